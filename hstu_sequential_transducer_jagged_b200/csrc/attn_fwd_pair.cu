// attn_fwd_pair.cu — jagged HSTU pointwise attention forward for head width 64 on the
// 5th-generation tensor cores: persistent CTAs, two query tiles per work item.
//
//   O_i = Σ_{j visible from i} SiLU(alpha <q_i, k_j> + rab_pos[..] + rab_time[..]) v_j
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, second formula; SiLU in place of
// softmax and no normalisation, "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 1; causal mask,
// or the M-FALCON candidate mask of §7.1.5.)
//
// With head width 64 the SiLU epilogue (one MUFU tanh per score) costs about as much as the two
// MMAs of a tile, so a work item holds two query tiles (256 rows of one sequence and head) that
// alternate: while epilogue warpgroup 0 turns S0 into P0, the tensor core runs PV1 and the next
// S1 for warpgroup 1, and the other way round.  Each K/V tile (and its 128 timestamps) is loaded
// once by TMA into a 4-stage ring and used by both query tiles.
//
// One CTA per SM walks the longest-first work list with a fixed stride (CTA b takes items
// b, b + grid, ...); barrier phases run on across items, so the producer streams the next
// item's tiles while the current one drains.  Warpgroup 0: warp 0 TMA producer; warp 1 TMEM
// allocation and single-thread tcgen05.mma issue (a thread that issues MMAs stalls for about
// their execution time, so issuing stays off the epilogue warps); warp 2 timestamps (per KV
// tile: min / max timestamp and int32 copies for the bias classification and gathers); warp 3
// spare.  Warpgroups 1 and 2: the two epilogue warpgroups (warp w owns TMEM lanes
// 32*(w%4) .. +31: one query row per thread).  After set-up warpgroup 0 gives registers to the
// epilogue warpgroups (setmaxnreg 88 / 208).
// TMEM (512 columns): S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384) O0 [384,448)
// O1 [448,512); P is bf16, two per 32-bit column, and feeds the PV MMA as its A operand.
//
// The relative bias rab_pos[clamp(p_i - p_j)] + rab_time[bucket(t_i - t_j)] is formed per row
// segment (one row, one KV tile): constant when every key falls in one position bucket (beyond
// the clamp) and one log2 time bucket (known from the tile's min/max timestamp, exact for any
// timestamp order because the bucket rule is monotone); else the position term comes from a
// 4-wide shifted copy of the table (one 16-byte shared load per 4 scores) and the time term
// from a threshold compare when the segment spans two buckets, or per element otherwise.
// Segments that cross the causal diagonal or hold candidates take the masked path.
#include <climits>

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kD = 64;
constexpr int kStages = 4;
constexpr int kThreads = 384;
constexpr int kTileBytes = kTileRows * kD * 2;  // 16 KB bf16 tile, 128-byte swizzle
constexpr int kTsBox = 136;      // timestamps loaded per KV tile (x rounded down to even)
constexpr int kTsStride = 144;   // per-stage buffer: 1152 bytes keeps every TMA destination 128-byte aligned
constexpr int kTimeSmem = 64;

__device__ __forceinline__ uint32_t col_s(int a) { return 128u * a; }
__device__ __forceinline__ uint32_t col_p(int a) { return 256u + 64u * a; }
__device__ __forceinline__ uint32_t col_o(int a) { return 384u + 64u * a; }

struct PairSmem {
  // every TMA destination below is 128-byte aligned (tiles 1024, timestamp stages 1152 bytes)
  alignas(1024) uint8_t q[2][kTileBytes];
  alignas(1024) uint8_t k[kStages][kTileBytes];
  alignas(1024) uint8_t v[kStages][kTileBytes];
  alignas(128) long long ts[kStages][kTsStride];
  alignas(16) int ts32[kStages][kTileRows];  // low 32 bits of the tile's 128 timestamps
  float rab_time_h[kTimeSmem];  // 0.5 x rab_time, clamped index
  long long tmin[kStages];       // min / max timestamp of each stage's in-sequence columns
  long long tmax[kStages];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages];
  uint64_t ts_ready[kStages];    // ts32 / tmin / tmax of the stage published (warp 10)
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t p_full[2];
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  // followed by: float4 pos4[P+1] (16-byte aligned), float pos_h[2P+1]
};

static_assert((kTsStride * 8) % 128 == 0, "timestamp stages must keep 128-byte alignment");
static_assert(offsetof(PairSmem, ts) % 128 == 0, "timestamp buffer alignment");

// The KV tiles a pair of query tiles visits, in load order U: history tiles 0..nhm-1, then the
// diagonal tile of query tile 0 and/or 1 when it is needed.  Query tile a visits history tiles
// 0..r[a].nh-1 and its diagonal.  r[1].nh - r[0].nh <= 1, so a query tile's next tile is never
// more than two positions ahead in U (the producer, 4 stages ahead, always has it in flight).
struct PairPlan {
  int q[2];
  bool valid[2];
  KvRange r[2];
  int nhm;
  int diag_u[2];
  int nU;

  __device__ __forceinline__ int tile_of(int u) const {
    return u < nhm ? u : (u == diag_u[0] ? q[0] : q[1]);
  }
  __device__ __forceinline__ bool member(int a, int u) const {
    if (!valid[a]) return false;
    return u < nhm ? (u < r[a].nh) : (u == diag_u[a]);
  }
  __device__ __forceinline__ int count(int a) const { return valid[a] ? r[a].count() : 0; }
  __device__ __forceinline__ int uidx(int a, int k) const { return k < r[a].nh ? k : diag_u[a]; }
};

__device__ __forceinline__ PairPlan make_plan(int qt0, int L, int n) {
  PairPlan p;
  p.q[0] = qt0;
  p.q[1] = qt0 + 1;
  p.valid[0] = qt0 * kTileRows < L;
  p.valid[1] = (qt0 + 1) * kTileRows < L;
  p.r[0] = kv_range(p.q[0], L, n);
  if (p.valid[1]) {
    p.r[1] = kv_range(p.q[1], L, n);
  } else {
    p.r[1].nh = 0;
    p.r[1].diag = 0;
  }
  p.nhm = max(p.r[0].nh, p.r[1].nh);
  int u = p.nhm;
  p.diag_u[0] = p.r[0].diag ? u++ : -1;
  p.diag_u[1] = p.r[1].diag ? u++ : -1;
  p.nU = u;
  return p;
}

__device__ __forceinline__ int clampi(int x, int lo, int hi) { return x < lo ? lo : (x > hi ? hi : x); }

// Waits for outstanding tcgen05.ld and ties the destination registers to the wait, so the
// compiler cannot read them before the data has landed.
__device__ __forceinline__ void tmem_wait_ld_regs(uint32_t (&r)[32]) {
  __syncwarp();
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]),
        "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]),
        "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
      :
      : "memory");
}

// floor(log2(max(1, d))) clamped to nb-1 for |d| < 2^23 without FLO: 2^23 + d is exact in
// fp32, so after subtracting 2^23 the exponent field is the bit length of d minus one.
__device__ __forceinline__ int bucket_small(int d, int nbm1) {
  d = d < 1 ? 1 : (d > 0x7FFFFF ? 0x7FFFFF : d);
  const float f = __int_as_float(0x4B000000 | d) - 8388608.0f;
  const int b = (__float_as_int(f) >> 23) - 127;
  return b < nbm1 ? b : nbm1;
}

// Per-row constants of one KV tile's epilogue.  The bias modes are warp-uniform (a warp takes
// a per-element path for all of its rows when any row needs it; the per-element formulas are
// exact for every row), so no branch inside the epilogue diverges.
struct RowCtx {
  float half_alpha;
  float half_bias;    // 0.5 x (the parts of the bias that are constant along the row segment)
  bool pos_elem;      // position term per element from the shifted table
  int t4_base;        // pos4 index of column c is clamp(t4_base - c, 0, P)
  int P;
  int time_mode;      // 0 constant, 1 threshold (row spans <= 2 buckets), 2 per element 32-bit,
                      // 3 per element 64-bit
  int thr;            // time_mode 1: dt >= thr takes t_hi
  float t_lo, t_hi;
  int ti_lo;
  long long ti;
  int pi_plus_p, P2, nbm1;
  int i, n, c0l;      // mask data (query index, history length, first column)
  bool row_valid;
  int mode;           // warp-uniform: 0 constant bias, 1 per-element bias, 2 masked
};

// 0.5 x rab_time of bucket(d) for |d| < 2^23 (table indexed by the biased fp32 exponent).
__device__ __forceinline__ float time_term32(const float* time_h, int d) {
  d = d < 1 ? 1 : (d > 0x7FFFFF ? 0x7FFFFF : d);
  const float f = __int_as_float(0x4B000000 | d) - 8388608.0f;
  return time_h[(__float_as_int(f) >> 23) - 127];
}

__device__ __forceinline__ float silu_half(float h) { return fmaf(h, tanh_fast(h), h); }

// One 32-column chunk: P = SiLU(alpha S + bias) as packed bf16.
template <int MODE>
__device__ __forceinline__ void silu_chunk(const uint32_t (&s)[32], uint32_t (&pk)[16], int ch,
                                           const RowCtx& rc, const float4* pos4,
                                           const float* pos_h, const float* time_h,
                                           const int* ts32, const long long* ts, bool use_pos,
                                           bool use_time) {
  if (MODE == 0) {
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      pk[e >> 1] = pack_bf16x2(silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e]), rc.half_bias)),
                               silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e + 1]), rc.half_bias)));
    return;
  }
#pragma unroll
  for (int e = 0; e < 32; e += 4) {
    const int c = ch * 32 + e;
    float b[4];
    if (MODE == 1) {
#pragma unroll
      for (int q = 0; q < 4; ++q) b[q] = rc.half_bias;
      if (rc.pos_elem) {
        const float4 pv = pos4[clampi(rc.t4_base - c, 0, rc.P)];
        b[0] += pv.x;
        b[1] += pv.y;
        b[2] += pv.z;
        b[3] += pv.w;
      }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        b[q] = 0.f;
        if (use_pos) {
          const int j = rc.c0l + c + q;  // candidate keys (j >= n) sit at position n
          b[q] = pos_h[clampi(rc.pi_plus_p - (j < rc.n ? j : rc.n), 0, rc.P2)];
        }
      }
    }
    if (rc.time_mode == 1) {
      const int4 tv = *reinterpret_cast<const int4*>(ts32 + c);
      b[0] += (rc.ti_lo - tv.x >= rc.thr) ? rc.t_hi : rc.t_lo;
      b[1] += (rc.ti_lo - tv.y >= rc.thr) ? rc.t_hi : rc.t_lo;
      b[2] += (rc.ti_lo - tv.z >= rc.thr) ? rc.t_hi : rc.t_lo;
      b[3] += (rc.ti_lo - tv.w >= rc.thr) ? rc.t_hi : rc.t_lo;
    } else if (rc.time_mode == 2) {
      const int4 tv = *reinterpret_cast<const int4*>(ts32 + c);
      b[0] += time_term32(time_h, rc.ti_lo - tv.x);
      b[1] += time_term32(time_h, rc.ti_lo - tv.y);
      b[2] += time_term32(time_h, rc.ti_lo - tv.z);
      b[3] += time_term32(time_h, rc.ti_lo - tv.w);
    } else if (rc.time_mode == 3) {
#pragma unroll
      for (int q = 0; q < 4; ++q) b[q] += time_h[time_bucket64(rc.ti - ts[c + q], rc.nbm1 + 1)];
    }
    float p[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      p[q] = silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e + q]), b[q]));
      if (MODE == 2) {
        const int j = rc.c0l + c + q;
        const bool vis = rc.row_valid && (j <= rc.i) && (j < rc.n || j == rc.i);
        p[q] = vis ? p[q] : 0.f;
      }
    }
    pk[e >> 1] = pack_bf16x2(p[0], p[1]);
    pk[(e >> 1) + 1] = pack_bf16x2(p[2], p[3]);
  }
}

// S (TMEM, this thread's row) -> P (TMEM, bf16) for one KV tile, loads software-pipelined.
template <int MODE>
__device__ __forceinline__ void tile_epilogue(uint32_t s_addr, uint32_t p_addr, const RowCtx& rc,
                                              const float4* pos4, const float* pos_h,
                                              const float* time_h, const int* ts32,
                                              const long long* ts, bool use_pos, bool use_time) {
  uint32_t b0[32], b1[32];
  uint32_t pk[16];
  tmem_ld32(s_addr, b0);
  tmem_wait_ld_regs(b0);
  tmem_ld32(s_addr + 32, b1);
  silu_chunk<MODE>(b0, pk, 0, rc, pos4, pos_h, time_h, ts32, ts, use_pos, use_time);
  tmem_st16(p_addr, pk);
  tmem_wait_ld_regs(b1);
  tmem_ld32(s_addr + 64, b0);
  silu_chunk<MODE>(b1, pk, 1, rc, pos4, pos_h, time_h, ts32, ts, use_pos, use_time);
  tmem_st16(p_addr + 16, pk);
  tmem_wait_ld_regs(b0);
  tmem_ld32(s_addr + 96, b1);
  silu_chunk<MODE>(b0, pk, 2, rc, pos4, pos_h, time_h, ts32, ts, use_pos, use_time);
  tmem_st16(p_addr + 32, pk);
  tmem_wait_ld_regs(b1);
  silu_chunk<MODE>(b1, pk, 3, rc, pos4, pos_h, time_h, ts32, ts, use_pos, use_time);
  tmem_st16(p_addr + 48, pk);
}

// S = Q Kᵀ for one 128 x 128 tile (4 MMAs of K = 16), completion signalled on bar.
__device__ __forceinline__ void issue_s_mma(uint32_t d_tmem, uint32_t qb, uint32_t kb,
                                            uint64_t* bar) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, 128, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk)
    mma_bf16_ss(d_tmem, smem_desc_sw128(qb + kk * 32, 16, 1024),
                smem_desc_sw128(kb + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  mma_commit(bar);
}

// O (+)= P V with P (bf16) read from TMEM and V (MN-major) from shared memory: 8 MMAs of K = 16.
__device__ __forceinline__ void issue_pv_mma(uint32_t o_tmem, uint32_t p_tmem, uint32_t vb,
                                             bool acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kD, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kTileRows / 16; ++kk)
    mma_bf16_ts(o_tmem, p_tmem + kk * 8, smem_desc_sw128(vb + kk * 2048, kTileRows * 128, 1024),
                idesc, (acc || kk > 0) ? 1u : 0u);
}

// Wait by one lane of the warp, then release the warp (the barrier's data is then visible to
// every lane: the waiting lane acquired it and the shuffle orders the warp's accesses).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// Bias classification of one row segment [c0l, c0l + 128) (this thread's query row; the
// stage's timestamps and their min / max must be published).  Returns the row context with the
// warp-uniform epilogue mode.  Everything is passed and returned by value so the context stays
// in registers.
__device__ __forceinline__ RowCtx classify_segment(RowCtx rc, int c0l, int i, int n, int pi,
                                                   long long ti, bool row_valid, bool use_pos,
                                                   bool use_time, int P, int NB,
                                                   long long tmin, long long tmax,
                                                   const float* pos_h, const float* time_h) {
  const int last = c0l + kTileRows - 1;
  const bool full_vis = last <= i && last < n;
  const bool need_mask = row_valid && !full_vis;
  const bool pos_elem = use_pos && row_valid && !(full_vis && pi - last >= P);
  bool fits32 = true, multi = false;
  int b_lo = 0, b_hi = 0;
  if (use_time) {
    const long long dt_lo = ti - tmax;
    const long long dt_hi = ti - tmin;
    fits32 = !row_valid || (dt_hi < (1ll << 23) && dt_lo > -(1ll << 23));
    b_lo = fits32 ? bucket_small(static_cast<int>(dt_lo), NB - 1) : time_bucket64(dt_lo, NB);
    b_hi = fits32 ? bucket_small(static_cast<int>(dt_hi), NB - 1) : time_bucket64(dt_hi, NB);
    multi = row_valid && b_hi > b_lo + 1;
  }
  const bool w_mask = __any_sync(0xffffffffu, need_mask);
  const bool w_pos = __any_sync(0xffffffffu, pos_elem);
  const bool w_tvar = __any_sync(0xffffffffu, row_valid && b_hi != b_lo);
  const bool w_multi = __any_sync(0xffffffffu, multi);
  const bool w_fits = __all_sync(0xffffffffu, fits32);
  float hbias = 0.f;
  if (use_pos && !w_pos) hbias = pos_h[2 * P];  // every valid row is beyond the clamp
  int tm = 0;
  if (use_time) {
    if (!w_tvar && !w_mask) {
      hbias += time_h[b_lo];                      // one bucket for every valid row
    } else if (!w_mask && !w_multi && w_fits) {
      tm = 1;                                     // at most two buckets per row
      rc.thr = 1 << (b_lo + 1);
      rc.t_lo = time_h[b_lo];
      rc.t_hi = time_h[b_hi];
    } else {
      tm = w_fits ? 2 : 3;
    }
  }
  rc.c0l = c0l;
  rc.pos_elem = w_pos;
  rc.t4_base = pi - c0l - 3;  // pos_base - (P + 3) with pos_base = pi - c0l + P
  rc.time_mode = tm;
  rc.half_bias = hbias;
  rc.mode = w_mask ? 2 : ((w_pos || tm != 0) ? 1 : 0);
  return rc;
}

// One query tile's MMAs for the current KV tile: wait for its P, (on the item's first tile) wait
// until the previous item's O was read, issue O (+)= P V, then the next S or the O commit.
__device__ __forceinline__ bool mma_step(PairSmem& sm, uint32_t tmem, const PairPlan& plan,
                                         int gu, int a, int st, int& pc, int& cnt, int oc,
                                         volatile int* abort_flag, int* status) {
  bool ok = mbar_wait(&sm.p_full[a], pc & 1, abort_flag, status);
  ++pc;
  if (ok && cnt == 0 && oc > 0) ok = mbar_wait(&sm.o_empty[a], (oc - 1) & 1, abort_flag, status);
  if (!ok) return false;
  tc_fence_after();
  issue_pv_mma(tmem + col_o(a), tmem + col_p(a), smem_u32(sm.v[st]), cnt > 0);
  ++cnt;
  if (cnt < plan.count(a)) {
    const int u2 = gu + plan.uidx(a, cnt);
    if (!mbar_wait(&sm.kv_full[u2 % kStages], (u2 / kStages) & 1, abort_flag, status)) return false;
    tc_fence_after();
    issue_s_mma(tmem + col_s(a), smem_u32(sm.q[a]), smem_u32(sm.k[u2 % kStages]), &sm.s_full[a]);
  } else {
    mma_commit(&sm.o_full[a]);
  }
  return true;
}

__device__ __forceinline__ void tma_load_1d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x)
      : "memory");
}

// 12 warps launch with 168 registers each (3 warps per SM sub-partition, 16K registers each);
// after set-up warpgroup 0 drops to 88 and the epilogue warpgroups rise to 208 (88 + 2 x 208 =
// 504 registers per sub-partition slot, the same 64512 the block launched with).
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                         const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_ts, AttnGeom g,
                         __nv_bfloat16* __restrict__ out, int64_t ld_o) {
  const int total = *g.item_count * g.H;
  if (static_cast<int>(blockIdx.x) >= total) return;
  if (*reinterpret_cast<volatile int*>(g.status) == kStatusTimeout) return;

  extern __shared__ uint8_t smem_raw[];
  PairSmem& sm = *reinterpret_cast<PairSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const bool use_time = (g.ts != nullptr) && (g.rab_time != nullptr);
  const bool use_pos = g.rab_pos != nullptr;  // the launcher guarantees P <= 2048
  float4* pos4 = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(&sm) + sizeof(PairSmem));
  float* pos_h = reinterpret_cast<float*>(pos4 + (use_pos ? g.P + 1 : 0));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- one-time setup: tables, barriers, TMEM
  if (use_pos) {
    const int P = g.P, P2 = 2 * g.P;
    for (int e = threadIdx.x; e <= P2; e += kThreads) pos_h[e] = 0.5f * g.rab_pos[e];
    // pos4[k] = 0.5 x (tab[x], tab[x-1], tab[x-2], tab[x-3]) with x = P + 3 + k, clamped at 2P
    for (int kx = threadIdx.x; kx <= P; kx += kThreads) {
      const int x = P + 3 + kx;
      pos4[kx] = make_float4(0.5f * g.rab_pos[min(x, P2)], 0.5f * g.rab_pos[min(x - 1, P2)],
                             0.5f * g.rab_pos[min(x - 2, P2)], 0.5f * g.rab_pos[min(x - 3, P2)]);
    }
  }
  if (use_time)
    for (int e = threadIdx.x; e < kTimeSmem; e += kThreads)
      sm.rab_time_h[e] = 0.5f * g.rab_time[e < g.NB ? e : g.NB - 1];
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.q_empty, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
      mbar_init(&sm.ts_ready[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.s_full[a], 1);
      mbar_init(&sm.p_full[a], 4);   // one elected lane per epilogue warp
      mbar_init(&sm.o_full[a], 1);
      mbar_init(&sm.o_empty[a], 4);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const int stride = static_cast<int>(gridDim.x);
  if (warp < 4) {
  setmaxnreg_dec<88>();
  if (warp == 0) {
    // ============================================================ producer
    if (lane == 0) {
      int gu = 0;  // KV tiles issued by this CTA so far
      int qi = 0;  // work items so far
      bool ok = true;
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      if (use_time) tma_prefetch_desc(&tm_ts);
      for (int w = blockIdx.x; ok && w < total; w += stride, ++qi) {
        const WorkItem it = g.items[w / g.H];
        const int head = w % g.H;
        const PairPlan plan =
            make_plan(it.qtile, it.len, hist_len(it.len, g.mask, g.num_candidates));
        if (qi > 0 && !mbar_wait(&sm.q_empty, (qi - 1) & 1, abort_flag, g.status)) {
          ok = false;
          break;
        }
        const int nq = plan.valid[1] ? 2 : 1;
        mbar_arrive_expect_tx(&sm.q_full, nq * kTileBytes);
        for (int a = 0; a < nq; ++a)
          tma_load_2d(sm.q[a], &tm_q, &sm.q_full, head * kD, it.row0 + plan.q[a] * kTileRows);
        for (int u = 0; u < plan.nU; ++u, ++gu) {
          const int st = gu % kStages;
          if (gu >= kStages &&
              !mbar_wait(&sm.kv_empty[st], ((gu / kStages) - 1) & 1, abort_flag, g.status)) {
            ok = false;
            break;
          }
          const int c0 = it.row0 + plan.tile_of(u) * kTileRows;
          mbar_arrive_expect_tx(&sm.kv_full[st], 2 * kTileBytes + (use_time ? kTsBox * 8 : 0));
          tma_load_2d(sm.k[st], &tm_k, &sm.kv_full[st], head * kD, c0);
          tma_load_2d(sm.v[st], &tm_v, &sm.kv_full[st], head * kD, c0);
          if (use_time) tma_load_1d(sm.ts[st], &tm_ts, &sm.kv_full[st], c0 & ~1);
        }
      }
      if (!ok) {  // leave no TMA write in flight into shared memory that is about to be released
        for (int u = (gu > kStages ? gu - kStages : 0); u < gu; ++u)
          mbar_wait(&sm.kv_full[u % kStages], (u / kStages) & 1, nullptr, nullptr);
        if (qi > 0) mbar_wait(&sm.q_full, (qi - 1) & 1, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ============================================================ MMA issuer
    if (lane == 0) {
      int gu = 0, qi = 0;
      int pc0 = 0, pc1 = 0;  // p_full phases consumed per query tile
      int oc0 = 0, oc1 = 0;  // items whose O was produced per query tile
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += stride, ++qi) {
        const WorkItem it = g.items[w / g.H];
        const PairPlan plan =
            make_plan(it.qtile, it.len, hist_len(it.len, g.mask, g.num_candidates));
        ok = mbar_wait(&sm.q_full, qi & 1, abort_flag, g.status);
        // first S of each query tile (the S buffers are free: the previous item's epilogue
        // finished reading them before its last p_full)
        for (int a = 0; ok && a < 2; ++a) {
          if (plan.count(a) == 0) continue;
          const int u = gu + plan.uidx(a, 0);
          ok = mbar_wait(&sm.kv_full[u % kStages], (u / kStages) & 1, abort_flag, g.status);
          if (ok) {
            tc_fence_after();
            issue_s_mma(tmem + col_s(a), smem_u32(sm.q[a]), smem_u32(sm.k[u % kStages]),
                        &sm.s_full[a]);
          }
        }
        int cnt0 = 0, cnt1 = 0;
        for (int u = 0; ok && u < plan.nU; ++u) {
          const int st = (gu + u) % kStages;
          if (plan.member(0, u)) ok = ok && mma_step(sm, tmem, plan, gu, 0, st, pc0, cnt0, oc0, abort_flag, g.status);
          if (plan.member(1, u)) ok = ok && mma_step(sm, tmem, plan, gu, 1, st, pc1, cnt1, oc1, abort_flag, g.status);
          if (!ok) break;
          mma_commit(&sm.kv_empty[st]);
        }
        if (plan.count(0) > 0) ++oc0;
        if (plan.count(1) > 0) ++oc1;
        gu += plan.nU;
        mma_commit(&sm.q_empty);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ============================================================ timestamp warp
    // For every KV tile the CTA loads: int32 copies of its 128 timestamps and the min / max
    // over its columns inside the sequence, published on ts_ready[stage].  A stage is refilled
    // only after both warpgroups' PV for it (after they used these values).
    if (use_time) {
      int gu = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += stride) {
        const WorkItem it = g.items[w / g.H];
        const PairPlan plan =
            make_plan(it.qtile, it.len, hist_len(it.len, g.mask, g.num_candidates));
        for (int u = 0; u < plan.nU; ++u, ++gu) {
          const int st = gu % kStages;
          ok = warp_wait(&sm.kv_full[st], (gu / kStages) & 1, abort_flag, g.status);
          if (!ok) break;
          const int c0l = plan.tile_of(u) * kTileRows;
          const long long* ts_tile = sm.ts[st] + ((it.row0 + c0l) & 1);
          long long mn = LLONG_MAX, mx = LLONG_MIN;
#pragma unroll
          for (int w4 = 0; w4 < kTileRows / 32; ++w4) {
            const int c = lane + 32 * w4;
            const long long tv = ts_tile[c];
            sm.ts32[st][c] = static_cast<int>(tv);
            if (c0l + c < it.len) {  // the sequence's own columns
              mn = tv < mn ? tv : mn;
              mx = tv > mx ? tv : mx;
            }
          }
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) {
            const long long omn = __shfl_xor_sync(0xffffffffu, mn, off);
            const long long omx = __shfl_xor_sync(0xffffffffu, mx, off);
            mn = omn < mn ? omn : mn;
            mx = omx > mx ? omx : mx;
          }
          if (lane == 0) {
            sm.tmin[st] = mn;
            sm.tmax[st] = mx;
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.ts_ready[st]);
        }
      }
    }
  }
  } else {
    setmaxnreg_inc<208>();
    // ============================================================ epilogue warpgroups
    const int a = (warp - 4) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    RowCtx rc;
    rc.half_alpha = 0.5f * g.alpha;
    rc.P = g.P;
    rc.P2 = 2 * g.P;
    rc.nbm1 = g.NB - 1;

    int gu = 0, sk = 0, oc = 0;
    bool ok = true;
    for (int w = blockIdx.x; ok && w < total; w += stride) {
      const WorkItem it = g.items[w / g.H];
      const int head = w % g.H;
      const int L = it.len;
      const int n = hist_len(L, g.mask, g.num_candidates);
      const PairPlan plan = make_plan(it.qtile, L, n);
      const int i = plan.q[a] * kTileRows + r;
      const bool row_valid = i < L;
      const int pi = i < n ? i : n;
      const long long ti = (use_time && row_valid) ? g.ts[it.row0 + i] : 0;
      rc.pi_plus_p = pi + g.P;
      rc.ti = ti;
      rc.ti_lo = static_cast<int>(ti);
      rc.i = i;
      rc.n = n;
      rc.row_valid = row_valid;
      const int cnt = plan.count(a);
      if (cnt > 0) {  // classify the first tile
        const int u = gu + plan.uidx(a, 0);
        if (use_time) ok = warp_wait(&sm.ts_ready[u % kStages], (u / kStages) & 1, abort_flag, g.status);
        if (!ok) break;
        const int st0 = u % kStages;
        rc = classify_segment(rc, plan.tile_of(plan.uidx(a, 0)) * kTileRows, i, n, pi, ti,
                              row_valid, use_pos, use_time, g.P, g.NB, sm.tmin[st0],
                              sm.tmax[st0], pos_h, sm.rab_time_h);
      }
      for (int k = 0; k < cnt; ++k, ++sk) {
        const int u = gu + plan.uidx(a, k);
        const int st = u % kStages;
        const long long* ts_tile = sm.ts[st] + ((it.row0 + rc.c0l) & 1);
        ok = warp_wait(&sm.s_full[a], sk & 1, abort_flag, g.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_addr = lane_addr + col_s(a);
        const uint32_t p_addr = lane_addr + col_p(a);
        // warp-uniform choice (tile_epilogue holds .sync.aligned TMEM loads/stores)
        if (rc.mode == 0)
          tile_epilogue<0>(s_addr, p_addr, rc, pos4, pos_h, sm.rab_time_h, sm.ts32[st], ts_tile,
                           use_pos, use_time);
        else if (rc.mode == 1)
          tile_epilogue<1>(s_addr, p_addr, rc, pos4, pos_h, sm.rab_time_h, sm.ts32[st], ts_tile,
                           use_pos, use_time);
        else
          tile_epilogue<2>(s_addr, p_addr, rc, pos4, pos_h, sm.rab_time_h, sm.ts32[st], ts_tile,
                           use_pos, use_time);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[a]);
        if (k + 1 < cnt) {  // classify the next tile while this tile's MMAs run
          const int u2 = gu + plan.uidx(a, k + 1);
          if (use_time)
            ok = warp_wait(&sm.ts_ready[u2 % kStages], (u2 / kStages) & 1, abort_flag, g.status);
          if (!ok) break;
          const int st2 = u2 % kStages;
          rc = classify_segment(rc, plan.tile_of(plan.uidx(a, k + 1)) * kTileRows, i, n, pi, ti,
                                row_valid, use_pos, use_time, g.P, g.NB, sm.tmin[st2],
                                sm.tmax[st2], pos_h, sm.rab_time_h);
        }
      }
      if (!ok) break;
      gu += plan.nU;
      if (cnt > 0) {
        // the item's output: wait for its last PV, read O from TMEM, store bf16 rows
        ok = warp_wait(&sm.o_full[a], oc & 1, abort_flag, g.status);
        if (!ok) break;
        ++oc;
        tc_fence_after();
        uint32_t o[32];
#pragma unroll 1
        for (int ch = 0; ch < kD / 32; ++ch) {
          tmem_ld32(lane_addr + col_o(a) + ch * 32, o);
          tmem_wait_ld_regs(o);
          if (row_valid) {
            uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(it.row0 + i) * ld_o +
                                                  head * kD + ch * 32);
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
              uint4 vv;
              vv.x = pack_bf16x2(__uint_as_float(o[8 * w4 + 0]), __uint_as_float(o[8 * w4 + 1]));
              vv.y = pack_bf16x2(__uint_as_float(o[8 * w4 + 2]), __uint_as_float(o[8 * w4 + 3]));
              vv.z = pack_bf16x2(__uint_as_float(o[8 * w4 + 4]), __uint_as_float(o[8 * w4 + 5]));
              vv.w = pack_bf16x2(__uint_as_float(o[8 * w4 + 6]), __uint_as_float(o[8 * w4 + 7]));
              dst[w4] = vv;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.o_empty[a]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

// Shared memory the paired kernel needs for position-table span P (0 when there is no table).
size_t attn_fwd_pair_smem(int P, bool has_pos) {
  size_t s = sizeof(PairSmem) + 1024;
  if (has_pos) s += sizeof(float4) * (P + 1) + sizeof(float) * (2 * P + 1);
  return s;
}

cudaError_t launch_attn_fwd_pair(const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& tts,
                                 const AttnGeom& g, __nv_bfloat16* out, int64_t ld_o, int grid,
                                 cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  const size_t smem = attn_fwd_pair_smem(g.P, g.rab_pos != nullptr);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_fwd_pair_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_fwd_pair_kernel<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tts, g, out, ld_o);
  return cudaGetLastError();
}

}  // namespace hstu
