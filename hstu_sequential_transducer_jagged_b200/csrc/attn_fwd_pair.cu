// attn_fwd_pair.cu — jagged HSTU pointwise attention forward for head width 64 on the
// 5th-generation tensor cores: persistent CTAs, two query tiles per work item, double-buffered
// scores.
//
//   O_i = Σ_{j visible from i} SiLU(alpha <q_i, k_j> + rab_pos[..] + rab_time[..]) v_j
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, second formula; SiLU in place of
// softmax and no normalisation, "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 1; causal mask,
// or the M-FALCON candidate mask of §7.1.5.)
//
// A work item is two 128-row query tiles of one sequence and head (Q double-buffered, so the
// next item's Q arrives while this one runs); keys and values stream through in 96-row tiles
// (TMA, 5-stage ring, the tile's timestamps with them) that both query tiles use.  Each query
// tile owns two 96-column score buffers in tensor memory and its epilogue writes P (bf16) over
// the S it has just read, so 2 x 2 x 96 + 2 x 64 (O) columns fit the 512 of an SM: while the
// epilogue turns S(k) into P(k), the tensor core already holds S(k+1), and S(k+2) is issued into
// the buffer of S(k) right after the PV that reads P(k) from it: tcgen05.mma instructions issued
// by one thread execute in order, so its writes follow that PV's reads without a wait (the
// pattern of the vendor's Blackwell attention, where each S buffer also holds P).
//
// Warpgroup 0: warp 0 TMA producer; warps 1 and 3 issue the tcgen05.mma of query tile 0 and 1
// (one thread each; warp 1 also owns the TMEM allocation); warp 2 classifies each KV tile (bias
// mode per segment, int32 timestamps, timestamp ranges) before its S is issued.  Warpgroups 1-4
// are the epilogue: warpgroup 1 + 2a + h handles query tile a, columns 48h .. 48h+47 of each
// score tile; warp w reads TMEM lanes 32 (w % 4) .. + 31, one query row per thread.  setmaxnreg
// moves registers from warpgroup 0 (64) to the epilogue warpgroups (104).
// TMEM (512 columns): score buffer b of query tile a at 96 (2a + b) (P of columns 48h.. at
// +48h, 24 columns of bf16 pairs), O of query tile a at 384 + 64 a.
//
// One CTA per SM walks the longest-first work list with a fixed stride; barrier phases run on
// across items (the S/P buffers alternate by a per-query-tile tile counter that never resets).
//
// The relative bias rab_pos[clamp(p_i - p_j)] + rab_time[bucket(t_i - t_j)] is formed per row
// segment (one row, one half of a KV tile): constant when every key is beyond the position clamp and in
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
constexpr int kKV = kPairKvRows;        // key/value tile rows (96)
constexpr int kSeg = 48;                // columns of a score tile per epilogue warp
constexpr int kStages = 5;
constexpr int kThreads = 640;          // 5 warpgroups
constexpr int kQBytes = kQ * kD * 2;    // 16 KB, 128-byte swizzle
constexpr int kKVBytes = kKV * kD * 2;  // 12 KB
constexpr int kTsBox = 98;              // timestamps loaded per KV tile (x rounded down to even)
constexpr int kTsStride = 112;          // 896-byte stages keep every TMA destination 128-aligned
constexpr int kTimeSmem = kTimeTableEntries;

__device__ __forceinline__ uint32_t col_buf(int a, int b) { return 96u * (2 * a + b); }
__device__ __forceinline__ uint32_t col_o(int a) { return 384u + 64u * a; }

struct PairSmem {
  alignas(1024) uint8_t q[2][2][kQBytes];  // [item slot][query tile]
  alignas(1024) uint8_t k[kStages][kKVBytes];
  alignas(1024) uint8_t v[kStages][kKVBytes];
  alignas(128) long long ts[kStages][kTsStride];
  alignas(16) int ts32[kStages][kKV];   // low 32 bits of the tile's timestamps
  float rab_time_h[kTimeSmem];           // 0.5 x rab_time, index clamped to NB - 1
  long long tmin[kStages][2];            // min / max timestamp of each 48-column half's
  long long tmax[kStages][2];            // in-sequence columns
  int2 cls[kStages][16];                 // per (query tile, row quarter, half): mode, bias
  uint64_t q_full[2], q_empty[2];        // per item slot
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t cls_ready[kStages];           // the tile's classification and timestamps
  uint64_t s_full[2][2];
  uint64_t p_full[2][2];
  uint64_t o_full[2];
  uint64_t o_empty[2];
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
  // followed by float4 pos4[2P + 4]: 0.5 x (tab[x], tab[x-1], tab[x-2], tab[x-3]), clamped
};

static_assert((kTsStride * 8) % 128 == 0, "timestamp stages must keep 128-byte alignment");
static_assert(kTsStride >= kTsBox, "timestamp stage holds one box");
static_assert(offsetof(PairSmem, ts) % 128 == 0, "timestamp buffer alignment");
static_assert(sizeof(PairSmem) % 16 == 0, "the position table follows the struct");
static_assert(kKVBytes % 1024 == 0, "K / V stages keep the 1024-byte swizzle alignment");
static_assert(kKV == 2 * kSeg && kSeg % 16 == 0, "two halves of 16-column chunks");

// KV tiles (96 rows) a 128-row query tile visits: history tiles 0..nh-1 (keys j < min(qe, n)),
// then nd (0..3) tiles from d0 on that hold the candidate rows' own keys beyond the history.
struct KvRangeP {
  int nh, d0, nd;
};

__device__ __forceinline__ KvRangeP kv_range_pair(int qt, int L, int n) {
  const int qs = qt * kQ;
  const int qe = min(qs + kQ, L);
  KvRangeP r;
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
// candidate tiles of query tile 0, then those of query tile 1.  A query tile's tiles are at
// most 5 positions apart in U.
struct PairPlan {
  int q[2];
  bool valid[2];
  KvRangeP r[2];
  int nhm;
  int base[2];  // U index of each query tile's first candidate tile
  int nU;

  __device__ __forceinline__ int tile_of(int u) const {
    if (u < nhm) return u;
    if (u < base[1]) return r[0].d0 + (u - base[0]);
    return r[1].d0 + (u - base[1]);
  }
  // (selects instead of indexing by a runtime a keep the plan in registers)
  __device__ __forceinline__ KvRangeP range(int a) const { return a == 0 ? r[0] : r[1]; }
  __device__ __forceinline__ int count(int a) const {
    const KvRangeP ra = range(a);
    return (a == 0 ? valid[0] : valid[1]) ? ra.nh + ra.nd : 0;
  }
  __device__ __forceinline__ int uidx(int a, int k) const {
    const KvRangeP ra = range(a);
    return k < ra.nh ? k : (a == 0 ? base[0] : base[1]) + (k - ra.nh);
  }
};

__device__ __forceinline__ PairPlan make_plan(int qt0, int L, int n) {
  PairPlan p;
  p.q[0] = qt0;
  p.q[1] = qt0 + 1;
  p.valid[0] = qt0 * kQ < L;
  p.valid[1] = (qt0 + 1) * kQ < L;
  p.r[0] = kv_range_pair(p.q[0], L, n);
  if (p.valid[1]) {
    p.r[1] = kv_range_pair(p.q[1], L, n);
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

// 0.5 x rab_time[bucket(d)] for |d| < 2^23 (the table holds clamped entries up to index 63).
__device__ __forceinline__ float time_term32(const float* time_h, int d) {
  return time_h[log2_small(d)];
}

// Per-row constants of one 48-column segment's epilogue.  The mode and the time-term kind are
// warp-uniform: a warp takes the per-element path for all of its rows when any row needs it
// (the per-element formulas are exact for every row), so no branch in the epilogue diverges.
struct RowCtx {
  float half_alpha;
  float half_bias;   // 0.5 x (the parts of the bias that are constant along the segment)
  int pbase;         // pos4 index of tile column c is clamp(pbase - c, 0, 2P+3)
  int time_mode;     // 0 constant, 1 threshold (<= 2 buckets), 2 per element 32-bit, 3 64-bit
  int thr;
  float t_lo, t_hi;
  int ti_lo;
  long long ti;
  int pi_plus_p, P2, nbm1;
  int i, n, c0t;     // query row, history length, first column of the KV tile
  bool row_valid;
  int mode;          // kModeConst, kModeElem, kModeCausal, kModeGeneral or kModeZero
};

constexpr int kModeConst = 0;    // one bias value per row
constexpr int kModeElem = 1;     // position term per element (+ time term), nothing masked
constexpr int kModeCausal = 2;   // as kModeElem, with the causal diagonal masked
constexpr int kModeGeneral = 3;  // M-FALCON candidates: everything per element, 64-bit time
constexpr int kModeZero = 4;     // every entry masked

// P = SiLU(alpha S + bias) for the W columns cb .. cb+W-1 of the tile, as packed bf16.
// TM is the time term's kind: 0 constant (in half_bias), 1 threshold, 2 per element from the
// 32-bit differences, 3 per element from the 64-bit differences.
template <int MODE, int TM, int W>
__device__ __forceinline__ void silu_chunk(const uint32_t (&s)[W], uint32_t (&pk)[W / 2], int cb,
                                           const RowCtx& rc, const float4* pos4,
                                           const float* time_h, const int* ts32,
                                           const long long* ts) {
#pragma unroll
  for (int q = 0; q < W; q += 4) {
    const int c = cb + q;  // column of the first of these 4 within the KV tile
    float bb[4];
    if (MODE == kModeConst) {
#pragma unroll
      for (int u = 0; u < 4; ++u) bb[u] = rc.half_bias;
    } else if (MODE == kModeElem || MODE == kModeCausal) {
      // exact for every row: beyond the band the clamped table repeats its last entry
      const float4 pv = pos4[pos4_row(rc.pbase, c, rc.P2)];
      const float2 hb = make_float2(rc.half_bias, rc.half_bias);
      const float2 b01 = add2(hb, make_float2(pv.x, pv.y));
      const float2 b23 = add2(hb, make_float2(pv.z, pv.w));
      bb[0] = b01.x;
      bb[1] = b01.y;
      bb[2] = b23.x;
      bb[3] = b23.y;
    } else {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = rc.c0t + c + u;  // candidate keys (j >= n) sit at position n
        bb[u] = pos4[pos4_general_row(rc.pi_plus_p, j, rc.n, rc.P2)].x;
      }
    }
    if (TM == 1 || TM == 2) {
      const int4 tv = *reinterpret_cast<const int4*>(ts32 + c);
      const int d[4] = {rc.ti_lo - tv.x, rc.ti_lo - tv.y, rc.ti_lo - tv.z, rc.ti_lo - tv.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        bb[u] += TM == 1 ? (threshold_takes_hi(d[u], rc.thr) ? rc.t_hi : rc.t_lo)
                         : time_term32(time_h, d[u]);
    } else if (TM == 3) {
#pragma unroll
      for (int u = 0; u < 4; ++u) bb[u] += time_h[time_bucket64(rc.ti - ts[c + u], rc.nbm1 + 1)];
    }
    // SiLU(x) = h (1 + tanh h), h = x / 2, on pairs of scores with packed f32x2 FMAs
    float p[4];
    const float2 ha = make_float2(rc.half_alpha, rc.half_alpha);
#pragma unroll
    for (int u = 0; u < 4; u += 2) {
      const float2 h = fma2(ha, make_float2(__uint_as_float(s[q + u]), __uint_as_float(s[q + u + 1])),
                            make_float2(bb[u], bb[u + 1]));
      const float2 pp = fma2(h, make_float2(tanh_fast(h.x), tanh_fast(h.y)), h);
      p[u] = pp.x;
      p[u + 1] = pp.y;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = rc.c0t + c + u;
      if (MODE == kModeCausal) p[u] = j <= rc.i ? p[u] : 0.f;
      if (MODE == kModeGeneral) {
        const bool vis = rc.row_valid && j <= rc.i && (j < rc.n || j == rc.i);
        p[u] = vis ? p[u] : 0.f;
      }
    }
    pk[q >> 1] = pack_bf16x2(p[0], p[1]);
    pk[(q >> 1) + 1] = pack_bf16x2(p[2], p[3]);
  }
}

__device__ __forceinline__ void tmem_wait_ld_regs16(uint32_t (&r)[16]) {
  __syncwarp();
  asm volatile(
      "tcgen05.wait::ld.sync.aligned;"
      : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]),
        "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]),
        "+r"(r[14]), "+r"(r[15])
      :
      : "memory");
}

// Each thread of a warp writes 8 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  __syncwarp();  // .sync.aligned: the whole warp, converged
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
      : "memory");
}

// This warp's 48 columns of S (TMEM) -> P (bf16, TMEM) in three 16-column chunks; the P of
// chunk c (8 columns of bf16 pairs) is written over columns 8c .. 8c+7, which belong to chunk
// 0 or 1 and have been read already.  One 16-column body per mode keeps the code small.
template <int MODE, int TM>
__device__ __forceinline__ void seg_epilogue(uint32_t seg_addr, int h, const RowCtx& rc,
                                             const float4* pos4, const float* time_h,
                                             const int* ts32, const long long* ts) {
#pragma unroll 1
  for (int c = 0; c < kSeg / 16; ++c) {
    uint32_t s[16];
    uint32_t pk[8];
    tmem_ld16(seg_addr + 16 * c, s);
    tmem_wait_ld_regs16(s);
    silu_chunk<MODE, TM, 16>(s, pk, kSeg * h + 16 * c, rc, pos4, time_h, ts32, ts);
    tmem_st8(seg_addr + 8 * c, pk);
  }
}

// Mode and bias of one (query tile, 32-row quarter, 48-column half) segment of a KV tile,
// decided by the classifier warp from the quarter's row ranges, so exact for every row: all
// entries masked (zero); a candidate row meeting candidate keys (general); keys past some row
// (causal diagonal); every key beyond the position clamp and every (row, key) pair in one time
// bucket (constant); else per element.  cls.x = mode | time-constant flag << 3, cls.y = 0.5 x
// the constant terms.
struct QuarterRows {
  int i0, i1;            // first and last valid row (i1 < i0: none)
  int pmin;              // smallest position among them
  long long tlo, thi;    // their timestamp range
};

__device__ __forceinline__ int2 classify_quarter(const QuarterRows& q, int c0, int n, int P,
                                                 bool use_pos, bool use_time, int NB,
                                                 long long tmin, long long tmax,
                                                 const float4* pos4, int P2,
                                                 const float* time_h) {
  const int last = c0 + kSeg - 1;
  int mode;
  if (q.i1 < q.i0 || c0 > q.i1) {
    mode = kModeZero;
  } else if (q.i1 >= n && last >= n) {
    mode = kModeGeneral;   // a candidate row meets candidate keys
  } else if (last > q.i0) {
    mode = kModeCausal;    // the causal diagonal (keys past the sequence are past it too)
  } else {
    mode = (use_pos && !pos_segment_beyond_clamp(q.pmin, last, P)) ? kModeElem : kModeConst;
  }
  bool tconst = true;
  float hb = 0.f;
  if (use_time && mode != kModeZero && mode != kModeGeneral) {
    // tmin / tmax cover the half's in-sequence keys, every key a row can see
    const int b_lo = time_bucket64(q.tlo - tmax, NB);
    const int b_hi = time_bucket64(q.thi - tmin, NB);
    tconst = b_lo == b_hi;
    if (tconst) hb = time_h[b_lo];
    else if (mode == kModeConst) mode = kModeElem;
  }
  if (mode == kModeConst) hb += pos4[P2 + 3].x;  // beyond the clamp: lane 0 reads entry 2P
  return make_int2(mode | (tconst ? 8 : 0), __float_as_int(hb));
}

// classify_quarter with the timestamps given relative to a common reference, all within
// +-2^30 of it, so the time buckets come from 32-bit differences (bucket32).
__device__ __forceinline__ int2 classify_quarter32(int i0, int i1, int pmin, int tlo, int thi,
                                                   int c0, int n, int P, bool use_pos,
                                                   bool use_time, int NB, int tmin, int tmax,
                                                   const float4* pos4, int P2,
                                                   const float* time_h) {
  const int last = c0 + kSeg - 1;
  int mode;
  if (i1 < i0 || c0 > i1) {
    mode = kModeZero;
  } else if (i1 >= n && last >= n) {
    mode = kModeGeneral;
  } else if (last > i0) {
    mode = kModeCausal;
  } else {
    mode = (use_pos && !pos_segment_beyond_clamp(pmin, last, P)) ? kModeElem : kModeConst;
  }
  bool tconst = true;
  float hb = 0.f;
  if (use_time && mode != kModeZero && mode != kModeGeneral) {
    const int b_lo = bucket32(tlo - tmax, NB - 1);
    const int b_hi = bucket32(thi - tmin, NB - 1);
    tconst = b_lo == b_hi;
    if (tconst) hb = time_h[b_lo];
    else if (mode == kModeConst) mode = kModeElem;
  }
  if (mode == kModeConst) hb += pos4[P2 + 3].x;
  return make_int2(mode | (tconst ? 8 : 0), __float_as_int(hb));
}

// The per-row part of a segment's set-up: the time term's kind when the quarter's rows do not
// share one bucket (threshold when every row spans at most two buckets, else per element), and
// the row constants.  Passed and returned by value so the context stays in registers.
__device__ __forceinline__ RowCtx segment_ctx(RowCtx rc, int2 cls, int c0t, int h, long long ti,
                                              bool row_valid, bool use_time, int NB,
                                              const long long* tmin, const long long* tmax,
                                              const float* time_h) {
  int mode = cls.x & 7;
  const bool tconst = (cls.x & 8) != 0;
  int tm = 0;
  if (use_time && !tconst) {
    const long long dt_lo = ti - *tmax;
    const long long dt_hi = ti - *tmin;
    const bool fits32 = !row_valid || (dt_hi < (1ll << 23) && dt_lo > -(1ll << 23));
    const bool w_fits = __all_sync(0xffffffffu, fits32);
    if (w_fits) {
      const int b_lo = bucket_small(static_cast<int>(dt_lo), NB - 1);
      const int b_hi = bucket_small(static_cast<int>(dt_hi), NB - 1);
      const bool w_multi = __any_sync(0xffffffffu, row_valid && b_hi > b_lo + 1);
      if (!w_multi) {
        tm = 1;
        rc.thr = threshold_of(b_lo);
        rc.t_lo = time_h[b_lo];
        rc.t_hi = time_h[b_hi];
      } else {
        tm = 2;
      }
    } else {
      tm = 3;
    }
  }
  if (mode == kModeGeneral) tm = use_time ? 3 : 0;
  // 64-bit differences: the general path (its visibility rule is exact for the causal mask too)
  if (tm == 3) mode = kModeGeneral;
  rc.c0t = c0t;
  rc.pbase = rc.pi_plus_p - c0t;
  rc.time_mode = tm;
  rc.half_bias = __int_as_float(cls.y);
  rc.mode = mode;
  return rc;
}

// Wait by one lane of the warp, then release the warp (the barrier's data is then visible to
// every lane: the waiting lane acquired it and the shuffle orders the warp's accesses).
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// warp_wait on two barriers; both probes are issued before either result is needed.
__device__ __forceinline__ bool warp_wait2(uint64_t* bar1, uint32_t parity1, uint64_t* bar2,
                                           uint32_t parity2, volatile int* abort, int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) {
    const bool p1 = mbar_try_wait(bar1, parity1);
    const bool p2 = mbar_try_wait(bar2, parity2);
    if (!p1) ok = mbar_wait(bar1, parity1, abort, status);
    if (ok && !p2) ok = mbar_wait(bar2, parity2, abort, status);
  }
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

// Issuer-side constants of one query tile: shared-memory descriptors of the first K and V
// stages and of the Q tile (a stage's descriptor adds stage x 512, the stage size >> 4), the
// tensor-memory columns, and the barriers.  Computed once so that the single issuing thread
// does no address arithmetic between MMAs.
struct IssuerCtx {
  uint64_t dq[2], dk0, dv0;        // dq per item slot
  uint32_t buf0, o_col;            // score buffer 1 lies 96 columns after buffer 0
  uint64_t* s_full0;               // buffer 1's barriers follow buffer 0's
  uint64_t* p_full0;
  uint64_t* o_full;
  uint64_t* o_empty;
  uint64_t* kv_full;
};

constexpr uint32_t kStageDesc = kKVBytes >> 4;  // descriptor step between K (or V) stages
static_assert(sizeof(PairSmem::k[0]) == kKVBytes && sizeof(PairSmem::v[0]) == kKVBytes,
              "K and V stages are contiguous");

__device__ __forceinline__ void issue_s(const IssuerCtx& c, uint64_t dq, int bs, int st) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kKV, 0, 0);
  const uint64_t dk = c.dk0 + static_cast<uint64_t>(st) * kStageDesc;
#pragma unroll
  for (int kk = 0; kk < kD / 16; ++kk)
    mma_bf16_ss(c.buf0 + 96u * bs, dq + 2 * kk, dk + 2 * kk, idesc, kk > 0 ? 1u : 0u);
  mma_commit(c.s_full0 + bs);
}

// O (+)= P V over the tile's 96 keys: P of keys 16kk.. is at column 8kk of the buffer for the
// first half and at 48 + 8 (kk - 3) for the second.
__device__ __forceinline__ void issue_pv(const IssuerCtx& c, int b, int st, bool acc) {
  constexpr uint32_t idesc = idesc_bf16_f32(128, kD, 0, 1);
  const uint64_t dv = c.dv0 + static_cast<uint64_t>(st) * kStageDesc;
  const uint32_t pb = c.buf0 + 96u * b;
#pragma unroll
  for (int kk = 0; kk < kKV / 16; ++kk)
    mma_bf16_ts(c.o_col, pb + (kk < 3 ? 8 * kk : 48 + 8 * (kk - 3)), dv + 128 * kk, idesc,
                (acc || kk > 0) ? 1u : 0u);
}

// 20 warps launch with 96 registers each (5 warps per SM sub-partition); after set-up
// warpgroup 0 drops to 64 and the four epilogue warpgroups rise to 104 (64 + 4 x 104 = 5 x 96).
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
  // (without a position table pos4 holds 4 zero entries, so the per-element path adds 0)
  const int P2 = use_pos ? 2 * g.P : 0;
  for (int x = threadIdx.x; x <= P2 + 3; x += kThreads)
    pos4[x] = use_pos ? make_float4(0.5f * g.rab_pos[pos4_lane_src(x, 0, P2)],
                                    0.5f * g.rab_pos[pos4_lane_src(x, 1, P2)],
                                    0.5f * g.rab_pos[pos4_lane_src(x, 2, P2)],
                                    0.5f * g.rab_pos[pos4_lane_src(x, 3, P2)])
                      : make_float4(0.f, 0.f, 0.f, 0.f);
  if (use_time)
    for (int e = threadIdx.x; e < kTimeSmem; e += kThreads)
      sm.rab_time_h[e] = 0.5f * g.rab_time[time_table_src(e, g.NB)];
  if (threadIdx.x == 0) {
    for (int sl = 0; sl < 2; ++sl) {
      mbar_init(&sm.q_full[sl], 1);
      mbar_init(&sm.q_empty[sl], 2);  // both issuers
    }
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 2);  // one release per query tile
      mbar_init(&sm.cls_ready[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      for (int b = 0; b < 2; ++b) {
        mbar_init(&sm.s_full[a][b], 1);
        mbar_init(&sm.p_full[a][b], 8);  // one elected lane per epilogue warp of tile a
      }
      mbar_init(&sm.o_full[a], 1);
      mbar_init(&sm.o_empty[a], 8);
    }
    mbar_init(&sm.drain[0], 1);
    mbar_init(&sm.drain[1], 1);
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
    setmaxnreg_dec<64>();
    if (warp == 0) {
      // ============================================================ producer
      if (lane == 0) {
        int gu = 0;  // KV tiles issued by this CTA so far
        int qi = 0;  // work items so far
        int qn = 0;  // Q loads issued
        bool ok = true;
        tma_prefetch_desc(&tm_q);
        tma_prefetch_desc(&tm_k);
        tma_prefetch_desc(&tm_v);
        if (use_time) tma_prefetch_desc(&tm_ts);
        WorkItem nxt = g.items[blockIdx.x / g.H];  // the next item is loaded one item ahead
        for (int w = blockIdx.x; ok && w < total; w += stride, ++qi) {
          const WorkItem it = nxt;
          if (w + stride < total) nxt = g.items[(w + stride) / g.H];
          const int head = w % g.H;
          const PairPlan plan =
              make_plan(it.qtile, it.len, hist_len(it.len, g.mask, g.num_candidates));
          const int sl = qi & 1;
          if (qi > 1 && !mbar_wait(&sm.q_empty[sl], ((qi >> 1) - 1) & 1, abort_flag, g.status)) {
            ok = false;
            break;
          }
          const int nq = plan.valid[1] ? 2 : 1;
          mbar_arrive_expect_tx(&sm.q_full[sl], nq * kQBytes);
          for (int a = 0; a < nq; ++a)
            tma_load_2d(sm.q[sl][a], &tm_q, &sm.q_full[sl], head * kD, it.row0 + plan.q[a] * kQ);
          ++qn;
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
          for (int q2 = (qn > 2 ? qn - 2 : 0); q2 < qn; ++q2)
            mbar_wait(&sm.q_full[q2 & 1], (q2 >> 1) & 1, nullptr, nullptr);
        }
      }
      __syncwarp();
    } else if (warp == 1 || warp == 3) {
      // ============================================================ MMA issuers
      // Query tile a's issuer walks every KV tile of each item in load order: for its own tiles
      // it issues PV and the S two tiles ahead; for the other tile's (candidate) tiles it waits
      // until the stage is loaded and releases it at once, so that neither side can release a
      // stage's next fill before its current one.  The epilogue of query tile a releases the
      // stages of its own tiles once their PV has completed.
      if (lane == 0) {
        const int a = warp == 1 ? 0 : 1;
        IssuerCtx c;
        c.dq[0] = smem_desc_sw128(smem_u32(sm.q[0][a]), 16, 1024);
        c.dq[1] = smem_desc_sw128(smem_u32(sm.q[1][a]), 16, 1024);
        c.dk0 = smem_desc_sw128(smem_u32(sm.k[0]), 16, 1024);
        c.dv0 = smem_desc_sw128(smem_u32(sm.v[0]), kKVBytes, 1024);
        c.buf0 = tmem + col_buf(a, 0);
        c.s_full0 = &sm.s_full[a][0];
        c.p_full0 = &sm.p_full[a][0];
        c.o_col = tmem + col_o(a);
        c.o_full = &sm.o_full[a];
        c.o_empty = &sm.o_empty[a];
        c.kv_full = sm.kv_full;
        int gu = 0, qi = 0, gs = 0, gp = 0, oc = 0;
        bool ok = true;
        WorkItem nxt = g.items[blockIdx.x / g.H];  // the next item is loaded one item ahead
        for (int w = blockIdx.x; ok && w < total; w += stride, ++qi) {
          const WorkItem it = nxt;
          if (w + stride < total) nxt = g.items[(w + stride) / g.H];
          const PairPlan plan =
              make_plan(it.qtile, it.len, hist_len(it.len, g.mask, g.num_candidates));
          // this query tile's KV tiles in load order: [0, nh) and [cb, ce)
          const KvRangeP rg = plan.range(a);
          const int cnt = plan.count(a);
          const int nh = cnt > 0 ? rg.nh : 0;
          const int cb = a == 0 ? plan.base[0] : plan.base[1];
          const int ce = cnt > 0 ? cb + rg.nd : cb;
          const int sl = qi & 1;
          const uint64_t dq = sl ? c.dq[1] : c.dq[0];
          ok = mbar_wait(&sm.q_full[sl], (qi >> 1) & 1, abort_flag, g.status);
          // prologue: the first two S (the buffers' previous P, of the last item, went to PVs
          // this thread has already issued, so in-order execution keeps them intact)
          const int first = ok ? min(2, cnt) : 0;
          for (int kk = 0; kk < first; ++kk) {
            const int u = gu + (kk < nh ? kk : cb + (kk - nh));
            // cls_ready follows kv_full: the classifier waited for the tile's load
            ok = mbar_wait(&sm.cls_ready[u % kStages], (u / kStages) & 1, abort_flag, g.status);
            if (!ok) break;
            tc_fence_after();
            issue_s(c, dq, gs & 1, u % kStages);
            ++gs;
          }
          int issued = first, done = 0;
          int st = gu % kStages, ph = (gu / kStages) & 1;  // stage and phase of tile u
          for (int u = 0; ok && u < plan.nU; ++u) {
            if (u < nh || (u >= cb && u < ce)) {
              const int b = gp & 1;
              ok = mbar_wait(c.p_full0 + b, (gp >> 1) & 1, abort_flag, g.status);
              ++gp;
              if (ok && done == 0 && oc > 0) ok = mbar_wait(c.o_empty, (oc - 1) & 1, abort_flag, g.status);
              if (!ok) break;
              tc_fence_after();
              issue_pv(c, b, st, done > 0);
              ++done;
              if (issued < cnt) {
                const int u2 = issued < nh ? issued : cb + (issued - nh);
                int st2 = st + (u2 - u), ph2 = ph;
                while (st2 >= kStages) {
                  st2 -= kStages;
                  ph2 ^= 1;
                }
                // into the buffer whose P the PV just issued reads: issued after it by this
                // thread, so executed after it
                ok = mbar_wait(&sm.cls_ready[st2], ph2, abort_flag, g.status);
                if (!ok) break;
                tc_fence_after();
                issue_s(c, dq, gs & 1, st2);
                ++gs;
                ++issued;
              }
              if (done == cnt) mma_commit(c.o_full);
            } else {
              ok = mbar_wait(&c.kv_full[st], ph, abort_flag, g.status);
              if (!ok) break;
              mbar_arrive(&sm.kv_empty[st]);
            }
            if (++st == kStages) {
              st = 0;
              ph ^= 1;
            }
          }
          if (cnt > 0) ++oc;
          gu += plan.nU;
          mma_commit(&sm.q_empty[sl]);
        }
        if (!ok) {  // every MMA this thread issued completes before TMEM is released
          mma_commit(&sm.drain[a]);
          mbar_wait(&sm.drain[a], 0, nullptr, nullptr);
        }
      }
      __syncwarp();
    } else if (warp == 2) {
      // ============================================================ classifier warp
      // For every KV tile the CTA loads: int32 copies of its timestamps, each 48-column half's
      // timestamp range over its in-sequence columns, and the mode and constant bias of the 16
      // (query tile, row quarter, half) segments, published on cls_ready[stage].  The issuers
      // wait for it before the tile's S, so an epilogue that has S has these too.  A stage is
      // refilled only after both query tiles released it, which follows their use of them.
      int gu = 0;
      bool ok = true;
      WorkItem nxt = g.items[blockIdx.x / g.H];  // the next item is loaded one item ahead
      for (int w = blockIdx.x; ok && w < total; w += stride) {
        const WorkItem it = nxt;
        if (w + stride < total) nxt = g.items[(w + stride) / g.H];
        const int L = it.len;
        const int n = hist_len(L, g.mask, g.num_candidates);
        const PairPlan plan = make_plan(it.qtile, L, n);
        // Row ranges of the 8 (query tile, quarter) groups.  Timestamps are taken relative to
        // t_ref (the item's first row) when every one the item touches lies within +-2^30 of it
        // (32-bit reductions), else the 64-bit path below runs.
        // lane s < 16 owns segment s = (query tile s >> 3, quarter s >> 1 & 3, half s & 1)
        const int grp = (lane >> 1) & 7;
        const int g_i0 = (plan.q[0] + (grp >> 2)) * kQ + 32 * (grp & 3);
        const int g_i1 = min(g_i0 + 31, L - 1);
        const int g_pmin = min(g_i0, n);
        long long t_ref = 0;
        bool rel32 = false;
        int g_tlo = 0, g_thi = 0;   // relative 32-bit row range of this lane's group
        QuarterRows qr;             // 64-bit row ranges (used when !rel32): lane c < 8: group c
        {
          const int c = lane & 7;
          qr.i0 = (plan.q[0] + (c >> 2)) * kQ + 32 * (c & 3);
          qr.i1 = min(qr.i0 + 31, L - 1);
          qr.pmin = min(qr.i0, n);
          qr.tlo = qr.thi = 0;
        }
        if (use_time) {
          // (t_ref is the first row of query tile 0; pass 1 checks the 32-bit range, pass 2
          // reduces; the row timestamps are read twice, the second time from cache)
          t_ref = g.ts[it.row0 + plan.q[0] * kQ];
          bool fits = true;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int i = (plan.q[0] + (c >> 2)) * kQ + 32 * (c & 3) + lane;
            const long long r64 = (i < L ? __ldg(&g.ts[it.row0 + i]) : t_ref) - t_ref;
            fits = fits && r64 < (1ll << 30) && r64 > -(1ll << 30);
          }
          rel32 = __all_sync(0xffffffffu, fits);
#pragma unroll 2
          for (int c = 0; c < 8; ++c) {
            const int i = (plan.q[0] + (c >> 2)) * kQ + 32 * (c & 3) + lane;
            const bool v = i < L;
            const long long tv = v ? __ldg(&g.ts[it.row0 + i]) : t_ref;
            if (rel32) {
              const int r = static_cast<int>(tv - t_ref);
              const int mn = __reduce_min_sync(0xffffffffu, v ? r : INT_MAX);
              const int mx = __reduce_max_sync(0xffffffffu, v ? r : INT_MIN);
              if (grp == c) {
                g_tlo = mn;
                g_thi = mx;
              }
            } else {
              long long mn = v ? tv : LLONG_MAX, mx = v ? tv : LLONG_MIN;
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) {
                const long long omn = __shfl_xor_sync(0xffffffffu, mn, off);
                const long long omx = __shfl_xor_sync(0xffffffffu, mx, off);
                mn = omn < mn ? omn : mn;
                mx = omx > mx ? omx : mx;
              }
              if ((lane & 7) == c) {
                qr.tlo = mn;
                qr.thi = mx;
              }
            }
          }
        }
        QuarterRows mine;  // 64-bit path: this lane's group
        mine.i0 = g_i0;
        mine.i1 = g_i1;
        mine.pmin = g_pmin;
        mine.tlo = __shfl_sync(0xffffffffu, qr.tlo, grp);
        mine.thi = __shfl_sync(0xffffffffu, qr.thi, grp);
        for (int u = 0; u < plan.nU; ++u, ++gu) {
          const int st = gu % kStages;
          ok = warp_wait(&sm.kv_full[st], (gu / kStages) & 1, abort_flag, g.status);
          if (!ok) break;
          const int c0t = plan.tile_of(u) * kKV;
          const int hf = lane & 1;
          if (!use_time) {
            if (lane < 16)
              sm.cls[st][lane] = classify_quarter32(g_i0, g_i1, g_pmin, 0, 0, c0t + kSeg * hf, n,
                                                    use_pos ? g.P : 0, use_pos, false, g.NB, 0, 0,
                                                    pos4, P2, sm.rab_time_h);
          } else {
            const long long* ts_tile = sm.ts[st] + ((it.row0 + c0t) & 1);
            // lane l holds columns l, l + 32, l + 64; half 0 is columns 0..47, half 1 48..95
            long long tv[3];
            bool in_seq[3], fits = rel32;
#pragma unroll
            for (int r3 = 0; r3 < 3; ++r3) {
              const int c = lane + 32 * r3;
              tv[r3] = ts_tile[c];
              sm.ts32[st][c] = static_cast<int>(tv[r3]);
              in_seq[r3] = c0t + c < L;  // the sequence's own columns
              const long long r64 = tv[r3] - t_ref;
              fits = fits && (!in_seq[r3] || (r64 < (1ll << 30) && r64 > -(1ll << 30)));
            }
            if (__all_sync(0xffffffffu, fits)) {
              int mn0 = INT_MAX, mx0 = INT_MIN, mn1 = INT_MAX, mx1 = INT_MIN;
#pragma unroll
              for (int r3 = 0; r3 < 3; ++r3) {
                const int c = lane + 32 * r3;
                const int r = static_cast<int>(tv[r3] - t_ref);
                if (in_seq[r3]) {
                  if (c < kSeg) {
                    mn0 = min(mn0, r);
                    mx0 = max(mx0, r);
                  } else {
                    mn1 = min(mn1, r);
                    mx1 = max(mx1, r);
                  }
                }
              }
              mn0 = __reduce_min_sync(0xffffffffu, mn0);
              mx0 = __reduce_max_sync(0xffffffffu, mx0);
              mn1 = __reduce_min_sync(0xffffffffu, mn1);
              mx1 = __reduce_max_sync(0xffffffffu, mx1);
              if (lane < 2) {  // the epilogue's per-row refinement reads absolute values
                sm.tmin[st][lane] = t_ref + (lane == 0 ? mn0 : mn1);
                sm.tmax[st][lane] = t_ref + (lane == 0 ? mx0 : mx1);
              }
              if (lane < 16)
                sm.cls[st][lane] = classify_quarter32(g_i0, g_i1, g_pmin, g_tlo, g_thi,
                                                      c0t + kSeg * hf, n, use_pos ? g.P : 0,
                                                      use_pos, true, g.NB, hf ? mn1 : mn0,
                                                      hf ? mx1 : mx0, pos4, P2, sm.rab_time_h);
            } else {
              long long mn0 = LLONG_MAX, mx0 = LLONG_MIN, mn1 = LLONG_MAX, mx1 = LLONG_MIN;
#pragma unroll
              for (int r3 = 0; r3 < 3; ++r3) {
                const int c = lane + 32 * r3;
                if (in_seq[r3]) {
                  if (c < kSeg) {
                    mn0 = tv[r3] < mn0 ? tv[r3] : mn0;
                    mx0 = tv[r3] > mx0 ? tv[r3] : mx0;
                  } else {
                    mn1 = tv[r3] < mn1 ? tv[r3] : mn1;
                    mx1 = tv[r3] > mx1 ? tv[r3] : mx1;
                  }
                }
              }
#pragma unroll
              for (int off = 16; off > 0; off >>= 1) {
                const long long a0 = __shfl_xor_sync(0xffffffffu, mn0, off);
                const long long b0 = __shfl_xor_sync(0xffffffffu, mx0, off);
                const long long a1 = __shfl_xor_sync(0xffffffffu, mn1, off);
                const long long b1 = __shfl_xor_sync(0xffffffffu, mx1, off);
                mn0 = a0 < mn0 ? a0 : mn0;
                mx0 = b0 > mx0 ? b0 : mx0;
                mn1 = a1 < mn1 ? a1 : mn1;
                mx1 = b1 > mx1 ? b1 : mx1;
              }
              if (lane < 2) {
                sm.tmin[st][lane] = lane == 0 ? mn0 : mn1;
                sm.tmax[st][lane] = lane == 0 ? mx0 : mx1;
              }
              if (!rel32) {  // the row ranges are 64-bit too
              } else {
                mine.tlo = t_ref + g_tlo;
                mine.thi = t_ref + g_thi;
              }
              if (lane < 16)
                sm.cls[st][lane] = classify_quarter(mine, c0t + kSeg * hf, n, use_pos ? g.P : 0,
                                                    use_pos, true, g.NB, hf ? mn1 : mn0,
                                                    hf ? mx1 : mx0, pos4, P2, sm.rab_time_h);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.cls_ready[st]);
        }
      }
    }
  } else {
    setmaxnreg_inc<104>();
    // ============================================================ epilogue warpgroups
    // Warpgroup 1 + 2 a + h handles query tile a, columns 48 h .. 48 h + 47 of every score tile
    // and columns 32 h .. 32 h + 31 of O; warp w reads TMEM lanes 32 (w % 4) .. + 31: one query
    // row per thread.
    const int e = warp - 4;
    const int a = e >> 3;
    const int h = (e >> 2) & 1;
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const bool lead = h == 0 && quad == 0 && lane == 0;  // releases KV stages for tile a
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    RowCtx rc;
    rc.half_alpha = 0.5f * g.alpha;
    rc.P2 = P2;
    rc.nbm1 = g.NB - 1;
    rc.thr = 0;
    rc.t_lo = rc.t_hi = 0.f;
    int gu = 0, gk = 0, oc = 0;  // gk: this query tile's KV tiles so far (selects S/P buffers)
    bool ok = true;
    WorkItem nxt = g.items[blockIdx.x / g.H];  // the next item is loaded one item ahead
    long long ti_next = 0;                     // and this row's timestamp in it
    {
      const int n0 = hist_len(nxt.len, g.mask, g.num_candidates);
      const PairPlan p0 = make_plan(nxt.qtile, nxt.len, n0);
      const int i0 = (a == 0 ? p0.q[0] : p0.q[1]) * kQ + r;
      if (use_time && i0 < nxt.len) ti_next = g.ts[nxt.row0 + i0];
    }
    for (int w = blockIdx.x; ok && w < total; w += stride) {
      const WorkItem it = nxt;
      if (w + stride < total) nxt = g.items[(w + stride) / g.H];
      const int head = w % g.H;
      const int L = it.len;
      const int n = hist_len(L, g.mask, g.num_candidates);
      const PairPlan plan = make_plan(it.qtile, L, n);
      const int i = (a == 0 ? plan.q[0] : plan.q[1]) * kQ + r;
      const bool row_valid = i < L;
      const int pi = i < n ? i : n;
      const long long ti = ti_next;
      rc.pi_plus_p = pi + (use_pos ? g.P : 0);
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
        const int c0t = plan.tile_of(uk) * kKV;
        const long long* ts_tile = sm.ts[st] + ((it.row0 + c0t) & 1);
        const int b = gk & 1;
        // S(k) follows the tile's classification (its issuer waited for it); the probe of
        // cls_ready makes that ordering explicit at almost no cost
        ok = warp_wait2(&sm.s_full[a][b], (gk >> 1) & 1, &sm.cls_ready[st], (u / kStages) & 1,
                        abort_flag, g.status);
        if (!ok) break;
        rc = segment_ctx(rc, sm.cls[st][8 * a + 2 * quad + h], c0t, h, ti, row_valid, use_time,
                         g.NB, &sm.tmin[st][h], &sm.tmax[st][h], sm.rab_time_h);
        // S(k) is complete, and so is every MMA this tile's issuer issued before it, PV(k-2)
        // among them: tile k-2's stage is free for this query tile
        if (k >= 2 && lead) mbar_arrive(&sm.kv_empty[(gu + plan.uidx(a, k - 2)) % kStages]);
        tc_fence_after();
        const uint32_t seg_addr = lane_addr + col_buf(a, b) + kSeg * h;
        const int* ts32 = sm.ts32[st];
        // warp-uniform choice (the epilogues hold .sync.aligned TMEM loads / stores)
        if (rc.mode == kModeConst) {
          seg_epilogue<kModeConst, 0>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
        } else if (rc.mode == kModeElem) {
          if (rc.time_mode == 0)
            seg_epilogue<kModeElem, 0>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
          else if (rc.time_mode == 1)
            seg_epilogue<kModeElem, 1>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
          else
            seg_epilogue<kModeElem, 2>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
        } else if (rc.mode == kModeCausal && rc.time_mode == 0) {
          seg_epilogue<kModeCausal, 0>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
        } else if (rc.mode == kModeCausal && rc.time_mode == 1) {
          seg_epilogue<kModeCausal, 1>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
        } else if (rc.mode == kModeCausal && rc.time_mode == 2) {
          seg_epilogue<kModeCausal, 2>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
        } else if (rc.mode == kModeZero) {
          uint32_t pk[16];
#pragma unroll
          for (int z = 0; z < 16; ++z) pk[z] = 0u;
          tmem_st16(seg_addr, pk);
          uint32_t pk8[8];
#pragma unroll
          for (int z = 0; z < 8; ++z) pk8[z] = 0u;
          tmem_st8(seg_addr + 16, pk8);
        } else {  // M-FALCON candidates, or 64-bit time differences
          seg_epilogue<kModeGeneral, 3>(seg_addr, h, rc, pos4, sm.rab_time_h, ts32, ts_tile);
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full[a][b]);
      }
      if (!ok) break;
      if (use_time && w + stride < total) {  // the next item's row timestamp
        const int n2 = hist_len(nxt.len, g.mask, g.num_candidates);
        const PairPlan p2 = make_plan(nxt.qtile, nxt.len, n2);
        const int i2 = (a == 0 ? p2.q[0] : p2.q[1]) * kQ + r;
        ti_next = i2 < nxt.len ? g.ts[nxt.row0 + i2] : 0;
      }
      if (cnt > 0) {
        // the item's output: wait for its last PV, read this warpgroup's 32 columns of O from
        // TMEM, store them as bf16
        ok = warp_wait(&sm.o_full[a], oc & 1, abort_flag, g.status);
        if (!ok) break;
        ++oc;
        if (lead)  // every PV of the item has completed: release the last two tiles' stages
          for (int k = max(0, cnt - 2); k < cnt; ++k)
            mbar_arrive(&sm.kv_empty[(gu + plan.uidx(a, k)) % kStages]);
        tc_fence_after();
        uint32_t o[32];
        tmem_ld32(lane_addr + col_o(a) + 32 * h, o);
        tmem_wait_ld_regs(o);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(it.row0 + i) * ld_o +
                                                head * kD + 32 * h);
          uint4 vv[4];
#pragma unroll
          for (int w4 = 0; w4 < 4; ++w4) {
            vv[w4].x = pack_bf16x2(__uint_as_float(o[8 * w4 + 0]), __uint_as_float(o[8 * w4 + 1]));
            vv[w4].y = pack_bf16x2(__uint_as_float(o[8 * w4 + 2]), __uint_as_float(o[8 * w4 + 3]));
            vv[w4].z = pack_bf16x2(__uint_as_float(o[8 * w4 + 4]), __uint_as_float(o[8 * w4 + 5]));
            vv[w4].w = pack_bf16x2(__uint_as_float(o[8 * w4 + 6]), __uint_as_float(o[8 * w4 + 7]));
            dst[w4] = vv[w4];
          }
          if (g.o_stats != nullptr) {
            // mean and sum of squared deviations of the 32 stored (bf16) values: two passes
            float f[32];
#pragma unroll
            for (int w4 = 0; w4 < 4; ++w4) {
              const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&vv[w4]);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 fv = __bfloat1622float2(p2[e]);
                f[8 * w4 + 2 * e] = fv.x;
                f[8 * w4 + 2 * e + 1] = fv.y;
              }
            }
            float sm8[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 32; ++e) sm8[e & 3] += f[e];
            const float mean = ((sm8[0] + sm8[1]) + (sm8[2] + sm8[3])) * (1.f / 32.f);
            float q8[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const float dl = f[e] - mean;
              q8[e & 3] = fmaf(dl, dl, q8[e & 3]);
            }
            g.o_stats[static_cast<int64_t>(it.row0 + i) * (g.H * (kD / 32)) + head * (kD / 32) + h] =
                make_float2(mean, (q8[0] + q8[1]) + (q8[2] + q8[3]));
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.o_empty[a]);
      }
      gu += plan.nU;
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
  s += sizeof(float4) * (has_pos ? 2 * P + 4 : 4);
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
