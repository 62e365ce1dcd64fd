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
// item's tiles while the current one drains.  Warps: 0 TMA producer; 1 TMEM allocation;
// 2-5 warpgroup 0 and 6-9 warpgroup 1 (warp w owns TMEM lanes 32*(w%4) .. +31: one query row
// per thread).  Each warpgroup issues its own MMAs: after its 128 threads have written P (a
// named barrier), one elected thread issues O += P V and the next S = Q Kᵀ, so the hand-off
// costs a named barrier instead of two mbarrier round trips through a separate MMA warp.
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
constexpr int kThreads = 320;
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
  float rab_time_h[kTimeSmem];  // 0.5 x rab_time, clamped index
  long long tmin[kStages];       // min / max timestamp of each stage's in-range columns
  long long tmax[kStages];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages];
  uint64_t ts_ready[kStages];    // tmin / tmax of the stage published (warp 1)
  uint64_t kv_empty[kStages];
  uint64_t s_full[2];
  uint64_t o_full[2];
  uint64_t drain[2];
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
// the per-element path for all of its rows when any row needs it: the per-element formulas are
// exact for every row), so no branch inside the epilogue diverges.
struct RowCtx {
  float half_alpha;
  float half_bias;    // 0.5 x (the parts of the bias that are constant along the row segment)
  bool pos_elem;      // position term per element (shifted table; exact for visible rows)
  int t4_base;        // pos4 index of column c is clamp(t4_base - c, 0, P)
  int pi_plus_p;      // p_i + P
  int P, P2;
  int time_mode;      // 0 in half_bias, 1 per element on 32-bit differences, 2 on 64-bit ones
  int ti_lo;
  long long ti;
  int nbm1;
  int i, n, c0l;      // mask data (query index, history length, first column)
  bool row_valid;
  int mode;           // warp-uniform: 0 constant bias, 1 per-element bias, 2 masked
};

// hb[e] = 0.5 x bias of column ch*32+e of this row's segment (segments without a mask).
__device__ __forceinline__ void bias_visible(float (&hb)[32], int ch, const RowCtx& rc,
                                             const float4* pos4, const float* time_h,
                                             const long long* ts) {
#pragma unroll
  for (int e = 0; e < 32; ++e) hb[e] = rc.half_bias;
  if (rc.pos_elem) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const float4 pv = pos4[clampi(rc.t4_base - (ch * 32 + e), 0, rc.P)];
      hb[e] += pv.x;
      hb[e + 1] += pv.y;
      hb[e + 2] += pv.z;
      hb[e + 3] += pv.w;
    }
  }
  const int* ts_lo = reinterpret_cast<const int*>(ts);  // low word of each int64 (little endian)
  if (rc.time_mode == 1) {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      hb[e] += time_h[bucket_small(rc.ti_lo - ts_lo[2 * (ch * 32 + e)], rc.nbm1)];
  } else if (rc.time_mode == 2) {
#pragma unroll
    for (int e = 0; e < 32; ++e) hb[e] += time_h[time_bucket64(rc.ti - ts[ch * 32 + e], rc.nbm1 + 1)];
  }
}

// hb[e] for segments on the causal diagonal or with candidate keys: general per-element bias.
__device__ __forceinline__ void bias_masked(float (&hb)[32], int ch, const RowCtx& rc,
                                            const float* pos_h, const float* time_h,
                                            const long long* ts, bool use_pos, bool use_time) {
#pragma unroll
  for (int e = 0; e < 32; ++e) hb[e] = 0.f;
  if (use_pos) {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int j = rc.c0l + ch * 32 + e;  // candidate keys (j >= n) sit at position n
      hb[e] += pos_h[clampi(rc.pi_plus_p - (j < rc.n ? j : rc.n), 0, rc.P2)];
    }
  }
  if (use_time) {
    const int* ts_lo = reinterpret_cast<const int*>(ts);
    if (rc.time_mode == 2) {
#pragma unroll
      for (int e = 0; e < 32; ++e) hb[e] += time_h[time_bucket64(rc.ti - ts[ch * 32 + e], rc.nbm1 + 1)];
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        hb[e] += time_h[bucket_small(rc.ti_lo - ts_lo[2 * (ch * 32 + e)], rc.nbm1)];
    }
  }
}

// One 32-column chunk: P = SiLU(alpha S + bias) as packed bf16.  MODE 0: constant bias;
// MODE 1: per-element bias without mask; MODE 2: masked segment.
template <int MODE>
__device__ __forceinline__ void silu_chunk(const uint32_t (&s)[32], uint32_t (&pk)[16], int ch,
                                           const RowCtx& rc, const float4* pos4,
                                           const float* pos_h, const float* time_h,
                                           const long long* ts, bool use_pos, bool use_time) {
  float hb[32];
  if (MODE == 0) {
#pragma unroll
    for (int e = 0; e < 32; ++e) hb[e] = rc.half_bias;
  } else if (MODE == 1) {
    bias_visible(hb, ch, rc, pos4, time_h, ts);
  } else {
    bias_masked(hb, ch, rc, pos_h, time_h, ts, use_pos, use_time);
  }
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float pv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float h = fmaf(rc.half_alpha, __uint_as_float(s[e + u]), hb[e + u]);
      float p = fmaf(h, tanh_fast(h), h);
      if (MODE == 2) {
        const int j = rc.c0l + ch * 32 + e + u;
        const bool vis = rc.row_valid && (j <= rc.i) && (j < rc.n || j == rc.i);
        p = vis ? p : 0.f;
      }
      pv[u] = p;
    }
    pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
  }
}

// S (TMEM, this thread's row) -> P (TMEM, bf16) for one KV tile, loads software-pipelined.
template <int MODE>
__device__ __forceinline__ void tile_epilogue(uint32_t s_addr, uint32_t p_addr, const RowCtx& rc,
                                              const float4* pos4, const float* pos_h,
                                              const float* time_h, const long long* ts,
                                              bool use_pos, bool use_time) {
  uint32_t b0[32], b1[32];
  uint32_t pk[16];
  tmem_ld32(s_addr, b0);
  tmem_wait_ld_regs(b0);
  tmem_ld32(s_addr + 32, b1);
  silu_chunk<MODE>(b0, pk, 0, rc, pos4, pos_h, time_h, ts, use_pos, use_time);
  tmem_st16(p_addr, pk);
  tmem_wait_ld_regs(b1);
  tmem_ld32(s_addr + 64, b0);
  silu_chunk<MODE>(b1, pk, 1, rc, pos4, pos_h, time_h, ts, use_pos, use_time);
  tmem_st16(p_addr + 16, pk);
  tmem_wait_ld_regs(b0);
  tmem_ld32(s_addr + 96, b1);
  silu_chunk<MODE>(b0, pk, 2, rc, pos4, pos_h, time_h, ts, use_pos, use_time);
  tmem_st16(p_addr + 32, pk);
  tmem_wait_ld_regs(b1);
  silu_chunk<MODE>(b1, pk, 3, rc, pos4, pos_h, time_h, ts, use_pos, use_time);
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

__device__ __forceinline__ void tma_load_1d(void* smem_dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3}], [%2];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x)
      : "memory");
}

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
    mbar_init(&sm.q_empty, 2);      // one commit per warpgroup and item
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 2);  // one commit per warpgroup (two from a sole user)
      mbar_init(&sm.ts_ready[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.s_full[a], 1);
      mbar_init(&sm.o_full[a], 1);
      mbar_init(&sm.drain[a], 1);
    }
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
    // ============================================================ timestamp statistics
    // For every KV tile the CTA loads: min / max timestamp of its columns inside the sequence,
    // published on ts_ready[stage] for the warpgroups' bias classification.  A stage is
    // refilled only after both warpgroups issued (and finished) their PV for it, which comes
    // after they read these values.
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
          const int c0 = it.row0 + c0l;
          const long long* ts_tile = sm.ts[st] + (c0 & 1);
          long long mn = LLONG_MAX, mx = LLONG_MIN;
#pragma unroll
          for (int w4 = 0; w4 < kTileRows / 32; ++w4) {
            const int c = lane + 32 * w4;
            if (c0l + c < it.len) {  // the sequence's own columns
              const long long tv = ts_tile[c];
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
  } else {
    // ============================================================ warpgroups 0 and 1
    const int a = (warp - 2) >> 2;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool leader = (warp == 2 + 4 * a) && lane == 0;  // issues this warpgroup's MMAs
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const uint32_t qb = smem_u32(sm.q[a]);
    const uint32_t s_tmem = tmem + col_s(a);
    const uint32_t p_tmem = tmem + col_p(a);
    const uint32_t o_tmem = tmem + col_o(a);
    RowCtx rc;
    rc.half_alpha = 0.5f * g.alpha;
    rc.P = g.P;
    rc.P2 = 2 * g.P;
    rc.nbm1 = g.NB - 1;
    int gu = 0, qi = 0, sk = 0, oc = 0;
    bool ok = true;

    // Bias classification of the row segment [c0l, c0l + 128) (KV tile uu of the item; the
    // timestamps of its stage must be ready).  Sets rc.{c0l, half_bias, pos_elem, t4_base,
    // time_mode, mode}.
    auto classify = [&](const PairPlan& plan, int uu, int st, int row0, int i, int n, int pi,
                        long long ti, bool row_valid) {
      const int c0l = plan.tile_of(uu) * kTileRows;
      const int last = c0l + kTileRows - 1;
      const bool full_vis = last <= i && last < n;
      const bool need_mask = row_valid && !full_vis;
      float hbias = 0.f;
      bool pos_elem = false, time_elem = false, fits32 = true;
      if (use_pos) pos_elem = row_valid && !(full_vis && pi - last >= g.P);
      int b_lo = 0;
      if (use_time) {
        const long long dt_lo = ti - sm.tmax[st];
        const long long dt_hi = ti - sm.tmin[st];
        fits32 = !row_valid || (dt_hi < (1ll << 23) && dt_lo > -(1ll << 23));
        b_lo = fits32 ? bucket_small(static_cast<int>(dt_lo), g.NB - 1) : time_bucket64(dt_lo, g.NB);
        const int b_hi = fits32 ? bucket_small(static_cast<int>(dt_hi), g.NB - 1)
                                : time_bucket64(dt_hi, g.NB);
        time_elem = row_valid && b_lo != b_hi;
      }
      const bool w_mask = __any_sync(0xffffffffu, need_mask);
      const bool w_pos = __any_sync(0xffffffffu, pos_elem);
      const bool w_time = __any_sync(0xffffffffu, time_elem);
      const bool w_fits = __all_sync(0xffffffffu, fits32);
      rc.c0l = c0l;
      rc.pos_elem = w_pos;
      rc.t4_base = pi - c0l - 3;  // pos_base - (P + 3) with pos_base = pi - c0l + P
      // constant parts: every valid row of a warp without per-element position terms is beyond
      // the clamp, and every valid row of a warp without per-element time terms has one bucket
      if (use_pos && !w_pos) hbias = pos_h[2 * g.P];
      rc.time_mode = w_time ? (w_fits ? 1 : 2) : 0;
      if (use_time && !w_time) hbias += sm.rab_time_h[b_lo];
      rc.half_bias = hbias;
      rc.mode = w_mask ? 2 : ((w_pos || w_time) ? 1 : 0);
      if (w_mask) rc.time_mode = w_fits ? 1 : 2;
    };

    // After a failed (timed-out) wait a warp keeps walking the loops "dry": it skips waits, TMEM
    // accesses and MMAs but still reaches every named barrier, so its siblings never block.
    for (int w = blockIdx.x; w < total; w += stride, ++qi) {
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
      // the item's first S (its Q tiles are loaded once the previous item released them)
      if (leader && ok) {
        ok = mbar_wait(&sm.q_full, qi & 1, abort_flag, g.status);
        if (ok && cnt > 0) {
          const int u = gu + plan.uidx(a, 0);
          ok = mbar_wait(&sm.kv_full[u % kStages], (u / kStages) & 1, abort_flag, g.status);
          if (ok) {
            tc_fence_after();
            issue_s_mma(s_tmem, qb, smem_u32(sm.k[u % kStages]), &sm.s_full[a]);
          }
        } else if (ok) {
          mbar_arrive(&sm.q_empty);  // this warpgroup has no rows in the item
        }
      }
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (cnt > 0) {  // classify the first tile
        const int u = gu + plan.uidx(a, 0);
        if (ok && use_time) ok = warp_wait(&sm.ts_ready[u % kStages], (u / kStages) & 1, abort_flag, g.status);
        classify(plan, plan.uidx(a, 0), u % kStages, it.row0, i, n, pi, ti, row_valid);
      }
      for (int k = 0; k < cnt; ++k, ++sk) {
        const int uu = plan.uidx(a, k);
        const int u = gu + uu;
        const int st = u % kStages;
        const long long* ts_tile = sm.ts[st] + ((it.row0 + rc.c0l) & 1);
        if (ok) ok = warp_wait(&sm.s_full[a], sk & 1, abort_flag, g.status);
        tc_fence_after();
        const uint32_t s_addr = lane_addr + col_s(a);
        const uint32_t p_addr = lane_addr + col_p(a);
        // warp-uniform choice (tile_epilogue holds .sync.aligned TMEM loads/stores)
        if (!ok) {
          // dry: nothing to compute
        } else if (rc.mode == 0)
          tile_epilogue<0>(s_addr, p_addr, rc, pos4, pos_h, sm.rab_time_h, ts_tile, use_pos,
                           use_time);
        else if (rc.mode == 1)
          tile_epilogue<1>(s_addr, p_addr, rc, pos4, pos_h, sm.rab_time_h, ts_tile, use_pos,
                           use_time);
        else
          tile_epilogue<2>(s_addr, p_addr, rc, pos4, pos_h, sm.rab_time_h, ts_tile, use_pos,
                           use_time);
        tmem_wait_st();
        tc_fence_before();
        named_barrier_sync(1 + a, 128);  // all of P (and every read of S) is done
        if (leader && ok) {
          tc_fence_after();
          issue_pv_mma(o_tmem, p_tmem, smem_u32(sm.v[st]), k > 0);
          mma_commit(&sm.kv_empty[st]);
          if (!plan.member(1 - a, uu)) mma_commit(&sm.kv_empty[st]);  // sole user of the tile
          if (k + 1 < cnt) {
            const int u2 = gu + plan.uidx(a, k + 1);
            ok = mbar_wait(&sm.kv_full[u2 % kStages], (u2 / kStages) & 1, abort_flag, g.status);
            if (ok) issue_s_mma(s_tmem, qb, smem_u32(sm.k[u2 % kStages]), &sm.s_full[a]);
          } else {
            mma_commit(&sm.o_full[a]);
            mma_commit(&sm.q_empty);
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
        if (k + 1 < cnt) {  // classify the next tile while this tile's MMAs run
          const int u2 = gu + plan.uidx(a, k + 1);
          if (ok && use_time)
            ok = warp_wait(&sm.ts_ready[u2 % kStages], (u2 / kStages) & 1, abort_flag, g.status);
          classify(plan, plan.uidx(a, k + 1), u2 % kStages, it.row0, i, n, pi, ti, row_valid);
        }
      }
      gu += plan.nU;
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (cnt > 0 && ok) ok = warp_wait(&sm.o_full[a], oc & 1, abort_flag, g.status);
      if (cnt > 0) ++oc;
      if (cnt > 0 && ok) {
        // the item's output: its last PV is done; read O from TMEM, store bf16 rows
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
      }
    }
    if (!ok && leader) {  // no MMA of this warpgroup may still be writing TMEM at the exit
      mma_commit(&sm.drain[a]);
      mbar_wait(&sm.drain[a], 0, nullptr, nullptr);
    }
    __syncwarp();
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
