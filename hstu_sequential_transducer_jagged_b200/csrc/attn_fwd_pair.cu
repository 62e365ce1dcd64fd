// attn_fwd_pair.cu — jagged HSTU pointwise attention forward for head width 64 on the
// 5th-generation tensor cores: persistent CTAs, two query tiles per work item, double-buffered
// scores.
//
//   O_i = Σ_{j visible from i} SiLU(alpha <q_i, k_j> + rab_pos[..] + rab_time[..]) v_j
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, second formula; SiLU in place of
// softmax and no normalisation, "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 1; causal mask,
// or the M-FALCON candidate mask of §7.1.5.)
//
// A work item is two 128-row query tiles of one sequence and head; keys and values stream
// through in 64-row tiles (TMA, 6-stage ring, the tile's timestamps with them) that both query
// tiles use.  Each query tile owns two S buffers and two P buffers in tensor memory: while its
// epilogue warpgroup turns S(k) into P(k), the tensor core already holds S(k+1), and S(k+2) is
// issued into the buffer S(k) leaves as soon as P(k) is written, so an epilogue warpgroup does
// not wait for the MMA chain and the two warpgroups keep the SFU (the SiLU's tanh) busy.
//
// Warpgroup 0: warp 0 TMA producer; warp 1 TMEM allocation and single-thread tcgen05.mma issue
// (a thread that issues MMAs stalls about as long as they execute, so issue stays off the
// epilogue warps); warp 2 timestamps (per KV tile: min / max and int32 copies); warp 3 spare.
// Warpgroups 1 and 2: one epilogue warpgroup per query tile (warp w owns TMEM lanes
// 32*(w%4) .. +31, one query row per thread).  setmaxnreg moves registers from warpgroup 0
// (88) to the epilogue warpgroups (208).
// TMEM (512 columns): S[a][b] at 64*(2a+b), P[a][b] (bf16 pairs) at 256 + 32*(2a+b),
// O[a] at 384 + 64*a, for query tile a and buffer b.
//
// One CTA per SM walks the longest-first work list with a fixed stride; barrier phases run on
// across items (the S/P buffers alternate by a per-query-tile tile counter that never resets).
//
// The relative bias rab_pos[clamp(p_i - p_j)] + rab_time[bucket(t_i - t_j)] is formed per row
// segment (one row, one KV tile): constant when every key is beyond the position clamp and in
// one log2 time bucket (from the tile's min / max timestamp; exact for any timestamp order since
// the bucket rule is monotone); else the position term comes from a 4-wide shifted table (one
// 16-byte shared load per 4 scores, exact with clamping at both ends) and the time term from a
// threshold when a row spans two buckets, or from the exponent of 2^23 + dt otherwise; tiles on
// the causal diagonal apply the mask in the same path.  Segments where a candidate row meets
// candidate keys (M-FALCON) take a general path.
#include <climits>
#include <cstddef>

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kD = 64;
constexpr int kQ = kTileRows;           // query tile rows (128)
constexpr int kKV = 64;                 // key/value tile rows
constexpr int kStages = 6;
constexpr int kThreads = 384;
constexpr int kQBytes = kQ * kD * 2;    // 16 KB, 128-byte swizzle
constexpr int kKVBytes = kKV * kD * 2;  // 8 KB
constexpr int kTsBox = 72;              // timestamps loaded per KV tile (x rounded down to even)
constexpr int kTsStride = 80;           // 640-byte stages keep every TMA destination 128-aligned
constexpr int kTimeSmem = 64;

__device__ __forceinline__ uint32_t col_s(int a, int b) { return 64u * (2 * a + b); }
__device__ __forceinline__ uint32_t col_p(int a, int b) { return 256u + 32u * (2 * a + b); }
__device__ __forceinline__ uint32_t col_o(int a) { return 384u + 64u * a; }

struct PairSmem {
  alignas(1024) uint8_t q[2][kQBytes];
  alignas(1024) uint8_t k[kStages][kKVBytes];
  alignas(1024) uint8_t v[kStages][kKVBytes];
  alignas(128) long long ts[kStages][kTsStride];
  alignas(16) int ts32[kStages][kKV];   // low 32 bits of the tile's timestamps
  float rab_time_h[kTimeSmem];           // 0.5 x rab_time, index clamped to NB - 1
  long long tmin[kStages];               // min / max timestamp of the tile's in-sequence columns
  long long tmax[kStages];
  uint64_t q_full, q_empty;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t ts_ready[kStages];
  uint64_t s_full[2][2];
  uint64_t p_full[2][2];
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  // followed by float4 pos4[2P + 4]: 0.5 x (tab[x], tab[x-1], tab[x-2], tab[x-3]), clamped
};

static_assert((kTsStride * 8) % 128 == 0, "timestamp stages must keep 128-byte alignment");
static_assert(kTsStride >= kTsBox, "timestamp stage holds one box");
static_assert(offsetof(PairSmem, ts) % 128 == 0, "timestamp buffer alignment");
static_assert(sizeof(PairSmem) % 16 == 0, "the position table follows the struct");

// KV tiles (64 rows) a 128-row query tile visits: history tiles 0..nh-1 (keys j < min(qe, n)),
// then nd (0..2) tiles from d0 on that hold the candidate rows' own keys beyond the history.
struct KvRange64 {
  int nh, d0, nd;
};

__device__ __forceinline__ KvRange64 kv_range64(int qt, int L, int n) {
  const int qs = qt * kQ;
  const int qe = min(qs + kQ, L);
  KvRange64 r;
  r.nh = (min(qe, n) + kKV - 1) / kKV;
  r.d0 = 0;
  r.nd = 0;
  if (qe > n) {
    r.d0 = max(r.nh, max(qs, n) / kKV);
    r.nd = max(0, (qe - 1) / kKV - r.d0 + 1);
  }
  return r;
}

// The KV tiles of a pair of query tiles, in load order U: history tiles 0..nhm-1, then the
// candidate tiles of query tile 0, then those of query tile 1.  A query tile's next tile is at
// most 4 positions ahead of its current one in U, inside the 6-stage ring.
struct PairPlan {
  int q[2];
  bool valid[2];
  KvRange64 r[2];
  int nhm;
  int base[2];  // U index of each query tile's first candidate tile
  int nU;

  __device__ __forceinline__ int tile_of(int u) const {
    if (u < nhm) return u;
    if (u < base[1]) return r[0].d0 + (u - base[0]);
    return r[1].d0 + (u - base[1]);
  }
  // (selects instead of indexing by a runtime a keep the plan in registers)
  __device__ __forceinline__ KvRange64 range(int a) const { return a == 0 ? r[0] : r[1]; }
  __device__ __forceinline__ bool member(int a, int u) const {
    const KvRange64 ra = range(a);
    const int ba = a == 0 ? base[0] : base[1];
    if (!(a == 0 ? valid[0] : valid[1])) return false;
    return u < nhm ? (u < ra.nh) : (u >= ba && u < ba + ra.nd);
  }
  __device__ __forceinline__ int count(int a) const {
    const KvRange64 ra = range(a);
    return (a == 0 ? valid[0] : valid[1]) ? ra.nh + ra.nd : 0;
  }
  __device__ __forceinline__ int uidx(int a, int k) const {
    const KvRange64 ra = range(a);
    return k < ra.nh ? k : (a == 0 ? base[0] : base[1]) + (k - ra.nh);
  }
};

__device__ __forceinline__ PairPlan make_plan(int qt0, int L, int n) {
  PairPlan p;
  p.q[0] = qt0;
  p.q[1] = qt0 + 1;
  p.valid[0] = qt0 * kQ < L;
  p.valid[1] = (qt0 + 1) * kQ < L;
  p.r[0] = kv_range64(p.q[0], L, n);
  if (p.valid[1]) {
    p.r[1] = kv_range64(p.q[1], L, n);
  } else {
    p.r[1].nh = 0;
    p.r[1].d0 = 0;
    p.r[1].nd = 0;
  }
  p.nhm = max(p.r[0].nh, p.r[1].nh);
  p.base[0] = p.nhm;
  p.base[1] = p.nhm + p.r[0].nd;
  p.nU = p.base[1] + p.r[1].nd;
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

// 0.5 x rab_time[bucket(d)] for |d| < 2^23 (the table holds clamped entries up to index 63).
__device__ __forceinline__ float time_term32(const float* time_h, int d) {
  d = d < 1 ? 1 : (d > 0x7FFFFF ? 0x7FFFFF : d);
  const float f = __int_as_float(0x4B000000 | d) - 8388608.0f;
  return time_h[(__float_as_int(f) >> 23) - 127];
}

__device__ __forceinline__ float silu_half(float h) { return fmaf(h, tanh_fast(h), h); }

// Per-row constants of one KV tile's epilogue.  The mode and the per-element switches are
// warp-uniform (a warp takes a per-element path for all of its rows when any row needs it; the
// per-element formulas are exact for every row), so no branch in the epilogue diverges.
struct RowCtx {
  float half_alpha;
  float half_bias;   // 0.5 x (the parts of the bias that are constant along the row segment)
  bool pos_elem;     // position term per element from pos4
  bool mask;         // causal mask inside the segment (diagonal tiles)
  int pbase;         // pos4 index of column c is clamp(pbase - c, 0, 2P+3)
  int time_mode;     // 0 constant, 1 threshold (<= 2 buckets), 2 per element 32-bit, 3 64-bit
  int thr;
  float t_lo, t_hi;
  int ti_lo;
  long long ti;
  int pi_plus_p, P2, nbm1;
  int i, n, c0l;
  bool row_valid;
  int mode;          // 0 constant bias, 1 per-element bias (+ causal mask), 2 general
};

// 0.5 x bias of columns ch*32 .. ch*32+31 (modes 1 and 2).
template <int MODE>
__device__ __forceinline__ void chunk_bias(float (&b)[32], int ch, const RowCtx& rc,
                                           const float4* pos4, const float* time_h,
                                           const int* ts32, const long long* ts, bool use_pos) {
  if (MODE == 1) {
#pragma unroll
    for (int e = 0; e < 32; ++e) b[e] = rc.half_bias;
    if (rc.pos_elem) {
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 pv = pos4[clampi(rc.pbase - (ch * 32 + e), 0, rc.P2 + 3)];
        b[e] += pv.x;
        b[e + 1] += pv.y;
        b[e + 2] += pv.z;
        b[e + 3] += pv.w;
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      b[e] = 0.f;
      if (use_pos) {
        const int j = rc.c0l + ch * 32 + e;  // candidate keys (j >= n) sit at position n
        b[e] = pos4[clampi(rc.pi_plus_p - (j < rc.n ? j : rc.n), 0, rc.P2)].x;
      }
    }
  }
  if (rc.time_mode == 1) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const int4 tv = *reinterpret_cast<const int4*>(ts32 + ch * 32 + e);
      b[e] += (rc.ti_lo - tv.x >= rc.thr) ? rc.t_hi : rc.t_lo;
      b[e + 1] += (rc.ti_lo - tv.y >= rc.thr) ? rc.t_hi : rc.t_lo;
      b[e + 2] += (rc.ti_lo - tv.z >= rc.thr) ? rc.t_hi : rc.t_lo;
      b[e + 3] += (rc.ti_lo - tv.w >= rc.thr) ? rc.t_hi : rc.t_lo;
    }
  } else if (rc.time_mode == 2) {
#pragma unroll
    for (int e = 0; e < 32; e += 4) {
      const int4 tv = *reinterpret_cast<const int4*>(ts32 + ch * 32 + e);
      b[e] += time_term32(time_h, rc.ti_lo - tv.x);
      b[e + 1] += time_term32(time_h, rc.ti_lo - tv.y);
      b[e + 2] += time_term32(time_h, rc.ti_lo - tv.z);
      b[e + 3] += time_term32(time_h, rc.ti_lo - tv.w);
    }
  } else if (rc.time_mode == 3) {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      b[e] += time_h[time_bucket64(rc.ti - ts[ch * 32 + e], rc.nbm1 + 1)];
  }
}

// One 32-column chunk: P = SiLU(alpha S + bias) as packed bf16, masked entries zero.
template <int MODE>
__device__ __forceinline__ void silu_chunk(const uint32_t (&s)[32], uint32_t (&pk)[16], int ch,
                                           const RowCtx& rc, const float4* pos4,
                                           const float* time_h, const int* ts32,
                                           const long long* ts, bool use_pos) {
  if (MODE == 0) {
#pragma unroll
    for (int e = 0; e < 32; e += 2)
      pk[e >> 1] =
          pack_bf16x2(silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e]), rc.half_bias)),
                      silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e + 1]), rc.half_bias)));
  } else {
    float b[32];
    chunk_bias<MODE>(b, ch, rc, pos4, time_h, ts32, ts, use_pos);
    if (MODE == 1 && !rc.mask) {
#pragma unroll
      for (int e = 0; e < 32; e += 2)
        pk[e >> 1] =
            pack_bf16x2(silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e]), b[e])),
                        silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e + 1]), b[e + 1])));
    } else {
#pragma unroll
      for (int e = 0; e < 32; e += 2) {
        float pv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int j = rc.c0l + ch * 32 + e + u;
          const float p = silu_half(fmaf(rc.half_alpha, __uint_as_float(s[e + u]), b[e + u]));
          bool vis = j <= rc.i;
          if (MODE == 2) vis = rc.row_valid && vis && (j < rc.n || j == rc.i);
          pv[u] = vis ? p : 0.f;
        }
        pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
      }
    }
  }
}

// S (TMEM, the 64 columns of this thread's row) -> P (TMEM, bf16); the second load overlaps the
// first chunk's math.
template <int MODE>
__device__ __forceinline__ void tile_epilogue(uint32_t s_addr, uint32_t p_addr, const RowCtx& rc,
                                              const float4* pos4, const float* time_h,
                                              const int* ts32, const long long* ts, bool use_pos) {
  uint32_t b0[32], b1[32];
  uint32_t pk[16];
  tmem_ld32(s_addr, b0);
  tmem_wait_ld_regs(b0);
  tmem_ld32(s_addr + 32, b1);
  silu_chunk<MODE>(b0, pk, 0, rc, pos4, time_h, ts32, ts, use_pos);
  tmem_st16(p_addr, pk);
  tmem_wait_ld_regs(b1);
  silu_chunk<MODE>(b1, pk, 1, rc, pos4, time_h, ts32, ts, use_pos);
  tmem_st16(p_addr + 16, pk);
}

// Bias classification of this thread's row segment [c0l, c0l + 64).  Passed and returned by
// value so the context stays in registers.
__device__ __forceinline__ RowCtx classify_segment(RowCtx rc, int c0l, int i, int n, int pi,
                                                   long long ti, bool row_valid, bool use_pos,
                                                   bool use_time, int P, int NB,
                                                   long long tmin, long long tmax,
                                                   const float4* pos4, const float* time_h) {
  const int last = c0l + kKV - 1;
  const bool cand = row_valid && i >= n && last >= n;  // a candidate row meets candidate keys
  const bool need_mask = row_valid && last > i;
  const bool pos_elem = use_pos && row_valid && !(pi - last >= P);
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
  const bool w_cand = __any_sync(0xffffffffu, cand);
  const bool w_mask = __any_sync(0xffffffffu, need_mask);
  const bool w_pos = __any_sync(0xffffffffu, pos_elem);
  const bool w_tvar = __any_sync(0xffffffffu, row_valid && b_hi != b_lo);
  const bool w_multi = __any_sync(0xffffffffu, multi);
  const bool w_fits = __all_sync(0xffffffffu, fits32);
  float hbias = 0.f;
  if (use_pos && !w_pos) hbias = pos4[2 * P].x;  // every valid row is beyond the clamp
  int tm = 0;
  if (use_time) {
    if (!w_tvar) {
      hbias += time_h[b_lo];                       // one bucket for each valid row
    } else if (!w_multi && w_fits) {
      tm = 1;                                      // at most two buckets per row
      rc.thr = 1 << (b_lo + 1);
      rc.t_lo = time_h[b_lo];
      rc.t_hi = time_h[b_hi];
    } else {
      tm = w_fits ? 2 : 3;
    }
  }
  rc.c0l = c0l;
  rc.pos_elem = w_pos;
  rc.mask = w_mask;
  rc.pbase = pi - c0l + P;
  rc.time_mode = tm;
  rc.half_bias = hbias;
  rc.mode = w_cand ? 2 : ((w_pos || w_mask || tm != 0) ? 1 : 0);
  if (rc.mode == 2) rc.time_mode = use_time ? (w_fits ? 2 : 3) : 0;
  return rc;
}

// S = Q Kᵀ for a 128 x 64 tile (4 MMAs of K = 16), completion signalled on bar.
__device__ __forceinline__ void issue_s_mma(uint32_t d_tmem, uint32_t qb, uint32_t kb,
                                            uint64_t* bar) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kKV, 0, 0);
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk)
    mma_bf16_ss(d_tmem, smem_desc_sw128(qb + kk * 32, 16, 1024),
                smem_desc_sw128(kb + kk * 32, 16, 1024), idesc, kk > 0 ? 1u : 0u);
  mma_commit(bar);
}

// O (+)= P V with P (bf16, 128 x 64) read from TMEM and V (MN-major) from shared memory.
__device__ __forceinline__ void issue_pv_mma(uint32_t o_tmem, uint32_t p_tmem, uint32_t vb,
                                             bool acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kD, 0, 1);
#pragma unroll
  for (int kk = 0; kk < kKV / 16; ++kk)
    mma_bf16_ts(o_tmem, p_tmem + kk * 8, smem_desc_sw128(vb + kk * 2048, kKVBytes, 1024), idesc,
                (acc || kk > 0) ? 1u : 0u);
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

// MMA-warp state of one query tile: S issued (gs) and P consumed (gp) in total (the buffers
// alternate across items), S issued and PV done in the current item, items with output (oc).
struct MmaTileState {
  int gs, gp, issued, done, oc;
};

// The PV of query tile a's current tile, then its S two tiles ahead (into the buffer just
// freed), and the output commit after its last tile.
__device__ __forceinline__ bool mma_step(PairSmem& sm, uint32_t tmem, const PairPlan& plan,
                                         int gu, int a, int st, MmaTileState& t,
                                         volatile int* abort_flag, int* status) {
  const int b = t.gp & 1;
  bool ok = mbar_wait(&sm.p_full[a][b], (t.gp >> 1) & 1, abort_flag, status);
  ++t.gp;
  if (ok && t.done == 0 && t.oc > 0)
    ok = mbar_wait(&sm.o_empty[a], (t.oc - 1) & 1, abort_flag, status);
  if (!ok) return false;
  tc_fence_after();
  issue_pv_mma(tmem + col_o(a), tmem + col_p(a, b), smem_u32(sm.v[st]), t.done > 0);
  ++t.done;
  if (t.issued < plan.count(a)) {
    const int u2 = gu + plan.uidx(a, t.issued);
    if (!mbar_wait(&sm.kv_full[u2 % kStages], (u2 / kStages) & 1, abort_flag, status)) return false;
    tc_fence_after();
    const int bs = t.gs & 1;
    issue_s_mma(tmem + col_s(a, bs), smem_u32(sm.q[a]), smem_u32(sm.k[u2 % kStages]),
                &sm.s_full[a][bs]);
    ++t.gs;
    ++t.issued;
  }
  if (t.done == plan.count(a)) mma_commit(&sm.o_full[a]);
  return true;
}

// 12 warps launch with 168 registers each (3 warps per SM sub-partition); after set-up
// warpgroup 0 drops to 88 and the epilogue warpgroups rise to 208 (88 + 2 x 208 = 3 x 168).
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

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- one-time setup: tables, barriers, TMEM
  if (use_pos) {
    const int P2 = 2 * g.P;
    for (int x = threadIdx.x; x <= P2 + 3; x += kThreads)
      pos4[x] = make_float4(0.5f * g.rab_pos[clampi(x, 0, P2)], 0.5f * g.rab_pos[clampi(x - 1, 0, P2)],
                            0.5f * g.rab_pos[clampi(x - 2, 0, P2)], 0.5f * g.rab_pos[clampi(x - 3, 0, P2)]);
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
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[a][b], 1);
        mbar_init(&sm.p_full[a][b], 4);  // one elected lane per epilogue warp
      }
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
          mbar_arrive_expect_tx(&sm.q_full, nq * kQBytes);
          for (int a = 0; a < nq; ++a)
            tma_load_2d(sm.q[a], &tm_q, &sm.q_full, head * kD, it.row0 + plan.q[a] * kQ);
          for (int u = 0; u < plan.nU; ++u, ++gu) {
            const int st = gu % kStages;
            if (gu >= kStages &&
                !mbar_wait(&sm.kv_empty[st], ((gu / kStages) - 1) & 1, abort_flag, g.status)) {
              ok = false;
              break;
            }
            const int c0 = it.row0 + plan.tile_of(u) * kKV;
            mbar_arrive_expect_tx(&sm.kv_full[st], 2 * kKVBytes + (use_time ? kTsBox * 8 : 0));
            tma_load_2d(sm.k[st], &tm_k, &sm.kv_full[st], head * kD, c0);
            tma_load_2d(sm.v[st], &tm_v, &sm.kv_full[st], head * kD, c0);
            if (use_time) tma_load_1d(sm.ts[st], &tm_ts, &sm.kv_full[st], c0 & ~1);
          }
        }
        if (!ok) {  // leave no TMA write in flight into shared memory about to be released
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
        MmaTileState t0{0, 0, 0, 0, 0}, t1{0, 0, 0, 0, 0};
        bool ok = true;
        for (int w = blockIdx.x; ok && w < total; w += stride, ++qi) {
          const WorkItem it = g.items[w / g.H];
          const PairPlan plan =
              make_plan(it.qtile, it.len, hist_len(it.len, g.mask, g.num_candidates));
          ok = mbar_wait(&sm.q_full, qi & 1, abort_flag, g.status);
          t0.issued = t0.done = t1.issued = t1.done = 0;
          // prologue: the first two S of each query tile (the epilogue read their buffers'
          // previous contents before the P that this warp has already consumed)
#pragma unroll
          for (int a = 0; a < 2; ++a) {
            MmaTileState& t = a == 0 ? t0 : t1;
            const int first = ok ? min(2, plan.count(a)) : 0;
            for (int kk = 0; ok && kk < first; ++kk) {
              const int u = gu + plan.uidx(a, kk);
              ok = mbar_wait(&sm.kv_full[u % kStages], (u / kStages) & 1, abort_flag, g.status);
              if (!ok) break;
              tc_fence_after();
              const int bs = t.gs & 1;
              issue_s_mma(tmem + col_s(a, bs), smem_u32(sm.q[a]), smem_u32(sm.k[u % kStages]),
                          &sm.s_full[a][bs]);
              ++t.gs;
              ++t.issued;
            }
          }
          for (int u = 0; ok && u < plan.nU; ++u) {
            const int st = (gu + u) % kStages;
            if (plan.member(0, u)) ok = mma_step(sm, tmem, plan, gu, 0, st, t0, abort_flag, g.status);
            if (ok && plan.member(1, u))
              ok = mma_step(sm, tmem, plan, gu, 1, st, t1, abort_flag, g.status);
            if (!ok) break;
            mma_commit(&sm.kv_empty[st]);
          }
          if (plan.count(0) > 0) ++t0.oc;
          if (plan.count(1) > 0) ++t1.oc;
          gu += plan.nU;
          mma_commit(&sm.q_empty);
        }
        if (!ok) {  // every MMA issued so far completes before TMEM is released
          mma_commit(&sm.drain);
          mbar_wait(&sm.drain, 0, nullptr, nullptr);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ============================================================ timestamp warp
      // For every KV tile the CTA loads: int32 copies of its 64 timestamps and the min / max
      // over its columns inside the sequence, published on ts_ready[stage].  A stage is refilled
      // only after both query tiles' PV for it, which follows their use of these values.
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
            const int c0l = plan.tile_of(u) * kKV;
            const long long* ts_tile = sm.ts[st] + ((it.row0 + c0l) & 1);
            long long mn = LLONG_MAX, mx = LLONG_MIN;
#pragma unroll
            for (int w2 = 0; w2 < kKV / 32; ++w2) {
              const int c = lane + 32 * w2;
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
    rc.P2 = 2 * g.P;
    rc.nbm1 = g.NB - 1;
    int gu = 0, gk = 0, oc = 0;  // gk: this query tile's KV tiles so far (selects S/P buffers)
    bool ok = true;
    for (int w = blockIdx.x; ok && w < total; w += stride) {
      const WorkItem it = g.items[w / g.H];
      const int head = w % g.H;
      const int L = it.len;
      const int n = hist_len(L, g.mask, g.num_candidates);
      const PairPlan plan = make_plan(it.qtile, L, n);
      const int i = (a == 0 ? plan.q[0] : plan.q[1]) * kQ + r;
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
      for (int k = 0; k < cnt; ++k, ++gk) {
        const int uk = plan.uidx(a, k);
        const int u = gu + uk;
        const int st = u % kStages;
        if (use_time) ok = warp_wait(&sm.ts_ready[st], (u / kStages) & 1, abort_flag, g.status);
        if (!ok) break;
        const int c0l = plan.tile_of(uk) * kKV;
        rc = classify_segment(rc, c0l, i, n, pi, ti, row_valid, use_pos, use_time, g.P, g.NB,
                              sm.tmin[st], sm.tmax[st], pos4, sm.rab_time_h);
        const long long* ts_tile = sm.ts[st] + ((it.row0 + c0l) & 1);
        const int b = gk & 1;
        ok = warp_wait(&sm.s_full[a][b], (gk >> 1) & 1, abort_flag, g.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_addr = lane_addr + col_s(a, b);
        const uint32_t p_addr = lane_addr + col_p(a, b);
        // warp-uniform choice (tile_epilogue holds .sync.aligned TMEM loads / stores)
        if (rc.mode == 0)
          tile_epilogue<0>(s_addr, p_addr, rc, pos4, sm.rab_time_h, sm.ts32[st], ts_tile, use_pos);
        else if (rc.mode == 1)
          tile_epilogue<1>(s_addr, p_addr, rc, pos4, sm.rab_time_h, sm.ts32[st], ts_tile, use_pos);
        else
          tile_epilogue<2>(s_addr, p_addr, rc, pos4, sm.rab_time_h, sm.ts32[st], ts_tile, use_pos);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[a][b]);
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

// Shared memory the paired kernel needs for position-table span P.
size_t attn_fwd_pair_smem(int P, bool has_pos) {
  size_t s = sizeof(PairSmem) + 1024;
  if (has_pos) s += sizeof(float4) * (2 * P + 4);
  return s;
}

// Rows of one K / V tile (the box height of the K and V tensor maps) and timestamps per tile
// load (the box of the timestamp map).
int attn_fwd_pair_kv_rows() { return kKV; }
int attn_fwd_pair_ts_box() { return kTsBox; }

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
