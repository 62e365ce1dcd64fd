// attn_bwd_tc.cu — jagged HSTU pointwise attention backward for head width 64 on the
// 5th-generation tensor cores (hstu_attention_backward's path for bf16 with 16-byte aligned rows;
// other shapes take the CUDA-core kernels).
//
// With S = alpha Q Kᵀ + rab on visible pairs, P = SiLU(S), O = P V and the output gradient dO
// (chain rule through "万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, second formula):
//   dV = Pᵀ dO,  dP = dO Vᵀ,  dS = dP ⊙ SiLU'(S),  SiLU'(x) = σ(x) (1 + x (1 - σ(x))),
//   dQ = alpha dS K,  dK = alpha dSᵀ Q,
//   d rab_pos[k] = Σ dS over pairs with clamped distance index k, d rab_time[b] likewise per time
//   bucket (the N×N rab backward that "6.2 HSTU的工程突破" §6.2.3 names as the RAB's cost).
//
// Key/value-stationary: a CTA takes a (sequence, head, 128-row key tile) item and walks the
// query tiles from the diagonal to the end of the sequence.  Per query tile:
//   Sᵀ = K Qᵀ and dPᵀ = V dOᵀ                       (smem x smem MMAs, M = keys, N = queries)
//   epilogue (one key row per thread): x = alpha s + bias, σ = 1/2 + tanh(x/2)/2, P = x σ,
//     dS = dP σ (1 + x (1 - σ)), 0 where the mask hides the pair; Pᵀ and (alpha dS)ᵀ as bf16
//     over the first half of each 32-query chunk's own Sᵀ / dPᵀ columns (a chunk is one warp's,
//     so no warp writes columns another still reads), (alpha dS)ᵀ also to shared memory (the
//     MN-major A operand of dQ); bias-table gradients: position bins of band blocks summed by
//     diagonal (DiagBins), otherwise summed in registers along runs of one table index and
//     added to shared-memory bins when the index changes (the time table's bins one copy per
//     lane, so that lanes ending runs of the same index together hit different banks)
//   dV += Pᵀ dO,  dK += (alpha dS)ᵀ Q                 (tensor-memory A operand)
//   dQ  = (alpha dS) K -> tensor memory; at the next step each epilogue warp stages its 32 rows
//     x 16 columns in shared memory and adds them to an fp32 accumulator in global memory with a
//     TMA reduction (the tile is complete by then: its MMAs were issued before the next step's
//     Sᵀ / dPᵀ, and one thread's MMAs execute in order; the next dQ is issued only after every
//     warp's p_full, which follows its drain).  Converted to bf16 after the kernel.  Rows of a
//     ragged last query tile hold exact zeros (their dS is zero), so the reduction may cover
//     rows of the next sequence.
// TMEM columns: Sᵀ 0..127, dPᵀ 128..255, dV 256..319, dK 320..383, dQ 384..447.
// Warps: 0 TMA producer, 1 MMA issuer (and the TMEM allocation), 2-17 epilogue (lane quarter
// w % 4, 32-query chunk (w - 2) / 4: four warps per SM sub-partition to hide the latency of the
// per-element chain).  18 warps, at most 5 on a sub-partition: 96 registers a thread.
// Items are visited in the reverse of the forward's longest-first order (which sorts by the
// number of key tiles a query tile visits), so that key tiles near the start of long sequences,
// which walk the most query tiles, start first.
#include <climits>

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {
namespace {

constexpr int kD = 64;
constexpr int kT = 128;
constexpr int kQStages = 2;
constexpr int kThreads = 576;   // 18 warps
constexpr int kEpiWarps = 16;
constexpr int kEpiFirst = 2;
constexpr int kTileBytes = kT * kD * 2;   // 16 KB
constexpr int kTsStride = 144;            // 1152 bytes per stage (TMA destination 128-aligned)
constexpr int kTsBox = 130;
constexpr uint32_t kColST = 0, kColDPT = 128, kColDV = 256, kColDK = 320, kColDQ = 384;

struct BwdSmem {
  alignas(1024) uint8_t k[kTileBytes];
  alignas(1024) uint8_t v[kTileBytes];
  alignas(1024) uint8_t q[kQStages][kTileBytes];
  alignas(1024) uint8_t dO[kQStages][kTileBytes];
  alignas(1024) uint8_t ds[2 * kTileBytes];      // [query half][key row][64 queries] SW128
  alignas(1024) uint8_t dqs[16][32 * 64];        // dQ staging: [epilogue warp][32 rows][16 fp32] SW64
  alignas(128) long long tq[kQStages][kTsStride];  // timestamps of the query tile
  uint64_t kv_full, kv_empty;
  uint64_t qd_full[kQStages], qd_empty[kQStages];
  uint64_t s_full, p_full, dq_last, acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
  // followed by float bins[2P+1 + NB]
};

__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
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

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          int* status) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, parity, abort, status);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ void tma_load_1d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x) {
  asm volatile(
      "cp.async.bulk.tensor.1d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x)
      : "memory");
}

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Bias-gradient run: sums dS in registers while the table index stays the same and adds the
// sum to the shared-memory bin when the index moves on.  Bin i sits at bins[i * stride]: the
// time table's bins are spread one copy per lane (stride 32, bins offset by the lane), so that
// the 32 lanes of a warp, which often end runs of the same index together, add to 32 banks
// instead of one address.
struct BinRun {
  int idx;
  float acc;
  int stride;
  __device__ __forceinline__ void add(float* bins, int i, float v) {
    if (i != idx) {
      if (idx >= 0) atomicAdd(&bins[idx * stride], acc);
      idx = i;
      acc = 0.f;
    }
    acc += v;
  }
  __device__ __forceinline__ void flush(float* bins) {
    if (idx >= 0) atomicAdd(&bins[idx * stride], acc);
    idx = -1;
    acc = 0.f;
  }
};

// Per-thread constants of one item: the thread's key row and the tables.
struct BwdRow {
  int jrow, pj, n, L;
  bool jvalid;
  long long tj;
};
struct BwdTabs {
  const float* pos;   // rab_pos copy in shared memory
  const float* time;  // rab_time copy
  float* bins_pos;    // gradient bins
  float* bins_time;
  float alpha;
  int P, NB;
  bool use_pos, use_time;
};

// Classes of a 32-query x 32-key block of one warp (warp-uniform): every pair hidden; every pair
// visible with one position bin and one time bucket; every pair visible with one time bucket;
// the same two with every distance inside the position band (diagonal bin sums, see DiagBins),
// the second also with per-element time buckets from 32-bit differences; anything else
// (per-element mask, bias and bins).
constexpr int kChunkGeneral = 0, kChunkTimeConst = 1, kChunkConst = 2, kChunkZero = 3,
              kChunkBandTC = 4, kChunkBandT32 = 5, kChunkBandTH = 6, kChunkBandT32M = 7;
// kChunkBandTH: as kChunkBandT32 with every pair in bucket b or b + 1 (ctidx = b): the bucket is
// b + 1 iff the difference is at least 2^(b+1), one compare per pair.
// kChunkBandT32M: the causal diagonal block of two history tiles (i0 == j0), pair (j, i) visible
// iff j <= i, otherwise as kChunkBandT32.

// Position-bin sums of a fully visible 32 x 32 block whose distances all lie inside the band:
// the pair (key j0 + l, query i0 + e) falls in diagonal e - l + 31 (0..62), i.e. bin
// i0 - j0 - 31 + P + (e - l + 31).  Lane m keeps diagonals m and m + 32: at column e the value of
// lane (e + 31 - m) mod 32 belongs to diagonal m when m >= e and to m + 32 otherwise, so one
// shuffle per column replaces a shared-memory atomic per element; 63 atomics close the block.
struct DiagBins {
  float lo, hi;
  __device__ __forceinline__ void add(int e, float v) {
    const int m = threadIdx.x & 31;
    const float w = __shfl_sync(0xffffffffu, v, (e - 1 - m) & 31);
    if (m >= e) lo += w; else hi += w;
  }
  __device__ __forceinline__ void flush(float* bins, int first_bin) {
    const int m = threadIdx.x & 31;
    atomicAdd(&bins[first_bin + m], lo);
    if (m < 31) atomicAdd(&bins[first_bin + 32 + m], hi);
    lo = hi = 0.f;
  }
};

__device__ __forceinline__ long long warp_min64(long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const long long o = __shfl_xor_sync(0xffffffffu, v, off);
    v = o < v ? o : v;
  }
  return v;
}
__device__ __forceinline__ long long warp_max64(long long v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const long long o = __shfl_xor_sync(0xffffffffu, v, off);
    v = o > v ? o : v;
  }
  return v;
}

// Range of the 32 query timestamps tq_c[0..31] of a block (lane l holds entry l): offsets from
// entry 0 (one broadcast load) reduced with redux.sync when they all fit in 32 bits, else the
// 64-bit shuffle reductions.
__device__ __forceinline__ void query_time_range(const long long* tq_c, long long& lo,
                                                 long long& hi) {
  const long long v = tq_c[threadIdx.x & 31];
  const long long base = tq_c[0];
  const long long d = v - base;
  if (__all_sync(0xffffffffu, d >= INT_MIN && d <= INT_MAX)) {
    const int di = static_cast<int>(d);
    lo = base + __reduce_min_sync(0xffffffffu, di);
    hi = base + __reduce_max_sync(0xffffffffu, di);
  } else {
    lo = warp_min64(v);
    hi = warp_max64(v);
  }
}

// Class of the block of queries i0 .. i0+31 and keys j0 .. j0+31.  tq_c: the block's query
// timestamps (lane l reads entry l); tj_lo / tj_hi: the warp's key timestamp range.  For the two
// constant classes it returns the constant bias terms (summed in the per-element path's order:
// position, then time) and their bins.  Exact for every pair: the bucket rule is monotone in the
// time difference and the position clamp in the distance.
__device__ __forceinline__ int chunk_class(int i0, int j0, int L, int n, const BwdTabs& t,
                                           const long long* tq_c, long long tj_lo,
                                           long long tj_hi, float& cbias, int& cpidx,
                                           int& ctidx) {
  const int j1 = j0 + 31;
  if (i0 >= L || j0 >= L || i0 + 31 < j0) return kChunkZero;
  // the diagonal block inside the history (both masks reduce to j <= i there)
  const bool diag = i0 == j0 && i0 + 31 < n && t.use_time;
  if (!(i0 >= j1 && i0 + 31 < L && j1 < n) && !diag) return kChunkGeneral;
  // every distance i - j of the block in [-P, P] and every query a history token: the position
  // index is i - j + P, no clamp
  const bool band =
      t.use_pos && i0 + 31 < n && i0 + 31 - j0 <= t.P && (!diag || j1 - i0 <= t.P);
  float tterm = 0.f;
  ctidx = 0;
  if (t.use_time) {
    long long tq_lo, tq_hi;
    query_time_range(tq_c, tq_lo, tq_hi);
    const int b_lo = time_bucket64(tq_lo - tj_hi, t.NB);
    const int b_hi = time_bucket64(tq_hi - tj_lo, t.NB);
    if (b_lo != b_hi) {
      // per-element buckets: from the 32-bit differences when all of them lie in (-2^23, 2^23)
      const bool small = tq_hi - tj_lo < (1ll << 23) && tq_lo - tj_hi > -(1ll << 23);
      if (!(small && (band || !t.use_pos))) return kChunkGeneral;
      ctidx = b_lo;
      if (diag) return kChunkBandT32M;
      return b_hi == b_lo + 1 ? kChunkBandTH : kChunkBandT32;
    }
    if (diag) return kChunkGeneral;
    ctidx = b_lo;
    tterm = t.time[b_lo];
  }
  cpidx = 0;
  if (t.use_pos) {
    // keys are history tokens (position = index); queries past the history sit at n
    if (!pos_segment_beyond_clamp(i0 < n ? i0 : n, j1, t.P)) {
      cbias = tterm;
      return band ? kChunkBandTC : kChunkTimeConst;
    }
    cpidx = 2 * t.P;  // every distance at or beyond the clamp
    cbias = t.pos[cpidx] + tterm;
    return kChunkConst;
  }
  cbias = tterm;
  return kChunkConst;
}

// W columns of a key row (half of a 32-query block): P and alpha dS (bf16 pairs) from S and dP,
// and the bias gradients.  i_first: query index of the first column; tq_c: its timestamps.
template <int V, int W>
__device__ __forceinline__ void bwd_chunk(const uint32_t (&s)[W], const uint32_t (&dp)[W],
                                          uint32_t (&pk)[W / 2], uint32_t (&dk)[W / 2], int i_first,
                                          const long long* tq_c, const BwdRow& r,
                                          const BwdTabs& t, float cbias, int cpidx, int ctidx,
                                          BinRun& run_p, BinRun& run_t) {
  float sum = 0.f;  // constant classes: the block's dS total for the constant bins
#pragma unroll
  for (int e = 0; e < W; e += 2) {
    float pv[2], dsa[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int i = i_first + e + u;
      float bias;
      int pidx = 0, bidx = 0;
      if (V == kChunkConst) {
        bias = cbias;
      } else {
        bias = 0.f;
        if (t.use_pos) {
          const int pi = i < r.n ? i : r.n;
          pidx = pos_index_direct(pi, r.pj, t.P);
          bias += t.pos[pidx];
        }
        if (V == kChunkTimeConst) {
          bias += cbias;
        } else if (t.use_time) {
          bidx = time_bucket64(tq_c[e + u] - r.tj, t.NB);
          bias += t.time[bidx];
        }
      }
      const float x = fmaf(t.alpha, __uint_as_float(s[e + u]), bias);
      const float sg = fmaf(0.5f, tanh_fast(0.5f * x), 0.5f);
      float p = x * sg;
      float dsv = __uint_as_float(dp[e + u]) * sg * fmaf(x, 1.f - sg, 1.f);
      if (V == kChunkGeneral) {
        const bool vis = r.jvalid && i < r.L && r.jrow <= i && (r.jrow < r.n || r.jrow == i);
        p = vis ? p : 0.f;
        dsv = vis ? dsv : 0.f;
        if (vis && t.use_pos) run_p.add(t.bins_pos, pidx, dsv);
        if (vis && t.use_time) run_t.add(t.bins_time, bidx, dsv);
      } else {
        if (V == kChunkTimeConst && t.use_pos) run_p.add(t.bins_pos, pidx, dsv);
        sum += dsv;
      }
      pv[u] = p;
      dsa[u] = t.alpha * dsv;
    }
    pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
    dk[e >> 1] = pack_bf16x2(dsa[0], dsa[1]);
  }
  if (V == kChunkConst && t.use_pos) run_p.add(t.bins_pos, cpidx, sum);
  if (V != kChunkGeneral && t.use_time) run_t.add(t.bins_time, ctidx, sum);
}

// W columns of a fully visible band block (classes kChunkBandTC, kChunkBandT32, kChunkBandTH): the
// same P and alpha dS as bwd_chunk, with the position bins summed by diagonal (dg) and, for
// kChunkBandT32 / kChunkBandTH, the time bucket of each pair from the low 32 bits of the two
// timestamps (every difference of the block lies in (-2^23, 2^23)); kChunkBandTH sums its two
// time bins in registers and adds them to two runs (run_t, run_t2).  eg0: block column of the first of the W queries; pb: this
// key row's position index for that query (i - j + P); tq_lo: the queries' timestamps as pairs
// of 32-bit words, low word first.
template <int V, int W, bool MASKED = false>
__device__ __forceinline__ void bwd_chunk_band(const uint32_t (&s)[W], const uint32_t (&dp)[W],
                                               uint32_t (&pk)[W / 2], uint32_t (&dk)[W / 2],
                                               int eg0, int pb, int jmi, const unsigned* tq_lo,
                                               unsigned tj_lo, const BwdTabs& t, float cbias,
                                               int ctidx, DiagBins& dg, BinRun& run_t,
                                               BinRun& run_t2) {
  float sum = 0.f;     // kChunkBandTC: the block's dS total for its one time bin
  float sum_hi = 0.f;  // kChunkBandTH: the dS total of bucket ctidx + 1 (sum: of ctidx)
  const int thr = V == kChunkBandTH ? threshold_of(ctidx) : 0;
  const float t_lo = V == kChunkBandTH ? t.time[ctidx] : 0.f;
  const float t_hi = V == kChunkBandTH ? t.time[ctidx + 1] : 0.f;
#pragma unroll
  for (int e = 0; e < W; e += 2) {
    float pv[2], dsa[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float bias = V == kChunkBandTC ? cbias : 0.f;
      if (t.use_pos) bias += t.pos[pb + e + u];
      int bidx = 0;
      bool upper = false;
      if (V == kChunkBandT32) {
        bidx = bucket_small(static_cast<int>(tq_lo[2 * (e + u)] - tj_lo), t.NB - 1);
        bias += t.time[bidx];
      } else if (V == kChunkBandTH) {
        upper = threshold_takes_hi(static_cast<int>(tq_lo[2 * (e + u)] - tj_lo), thr);
        bias += upper ? t_hi : t_lo;
      }
      const float x = fmaf(t.alpha, __uint_as_float(s[e + u]), bias);
      const float sg = fmaf(0.5f, tanh_fast(0.5f * x), 0.5f);
      float p = x * sg;
      float dsv = __uint_as_float(dp[e + u]) * sg * fmaf(x, 1.f - sg, 1.f);
      if (MASKED) {  // column e + u visible iff it is at least jmi (the key row's own query)
        const bool vis = e + u >= jmi;
        p = vis ? p : 0.f;
        dsv = vis ? dsv : 0.f;
      }
      if (t.use_pos) dg.add(eg0 + e + u, dsv);
      if (V == kChunkBandT32) {
        run_t.add(t.bins_time, bidx, dsv);
      } else if (V == kChunkBandTH) {
        sum += upper ? 0.f : dsv;
        sum_hi += upper ? dsv : 0.f;
      } else {
        sum += dsv;
      }
      pv[u] = p;
      dsa[u] = t.alpha * dsv;
    }
    pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
    dk[e >> 1] = pack_bf16x2(dsa[0], dsa[1]);
  }
  if (V == kChunkBandTC && t.use_time) run_t.add(t.bins_time, ctidx, sum);
  if (V == kChunkBandTH) {  // two runs, so that neither ends at every block
    run_t.add(t.bins_time, ctidx, sum);
    run_t2.add(t.bins_time, ctidx + 1, sum_hi);
  }
}

// Items: (sequence, 128-row key tile) from the work list built with one tile per item, times heads.
template <bool kFast>
__global__ void __launch_bounds__(kThreads, 1)
    attn_bwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v,
                       const __grid_constant__ CUtensorMap tm_do,
                       const __grid_constant__ CUtensorMap tm_ts,
                       const __grid_constant__ CUtensorMap tm_dq, AttnGeom g,
                       __nv_bfloat16* __restrict__ dk_out, int64_t ld_dk,
                       __nv_bfloat16* __restrict__ dv_out, int64_t ld_dv,
                       float* __restrict__ d_pos, float* __restrict__ d_time, SiluGradZ zg) {
  const int nitems = *g.item_count;
  const int total = nitems * g.H;
  if (static_cast<int>(blockIdx.x) >= total) return;
  extern __shared__ uint8_t smem_raw[];
  BwdSmem& sm = *reinterpret_cast<BwdSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  float* bins = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(&sm) + sizeof(BwdSmem));
  const bool use_pos = g.rab_pos != nullptr;
  const bool use_time = g.ts != nullptr && g.rab_time != nullptr;
  const int npos = use_pos ? 2 * g.P + 1 : 0;
  const int nbins = npos + (use_time ? g.NB : 0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int stride = static_cast<int>(gridDim.x);

  // bins[0, nbins): gradient bins (the time entries unused); then copies of the two bias
  // tables; then the time table's bins, 32 copies (entry b of lane l at b * 32 + l)
  float* tab_pos = bins + nbins;
  float* tab_time = tab_pos + npos;
  float* tbins = tab_pos + nbins;
  const int ntime = nbins - npos;
  for (int e = threadIdx.x; e < nbins; e += kThreads) {
    bins[e] = 0.f;
    tab_pos[e] = e < npos ? g.rab_pos[e] : g.rab_time[e - npos];
  }
  for (int e = threadIdx.x; e < 32 * ntime; e += kThreads) tbins[e] = 0.f;
  if (threadIdx.x == 0) {
    mbar_init(&sm.kv_full, 1);
    mbar_init(&sm.kv_empty, 1);
    for (int s = 0; s < kQStages; ++s) {
      mbar_init(&sm.qd_full[s], 1);
      mbar_init(&sm.qd_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, kEpiWarps);
    mbar_init(&sm.dq_last, 1);
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, kEpiWarps);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int gs = 0, jj = 0, kv_issued = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += stride, ++jj) {
        const WorkItem it = g.items[nitems - 1 - w / g.H];
        const int head = w % g.H, kt = it.qtile, L = it.len;
        const int nt = (L + kT - 1) / kT;
        if (jj > 0 && !mbar_wait(&sm.kv_empty, (jj - 1) & 1, abort_flag, g.status)) {
          ok = false;
          break;
        }
        ++kv_issued;
        mbar_arrive_expect_tx(&sm.kv_full, 2 * kTileBytes);
        tma_load_2d(sm.k, &tm_k, &sm.kv_full, head * kD, it.row0 + kt * kT);
        tma_load_2d(sm.v, &tm_v, &sm.kv_full, head * kD, it.row0 + kt * kT);
        for (int qt = kt; qt < nt; ++qt, ++gs) {
          const int st = gs % kQStages;
          if (gs >= kQStages &&
              !mbar_wait(&sm.qd_empty[st], ((gs / kQStages) - 1) & 1, abort_flag, g.status)) {
            ok = false;
            break;
          }
          const int r0 = it.row0 + qt * kT;
          mbar_arrive_expect_tx(&sm.qd_full[st], 2 * kTileBytes + (use_time ? kTsBox * 8 : 0));
          tma_load_2d(sm.q[st], &tm_q, &sm.qd_full[st], head * kD, r0);
          tma_load_2d(sm.dO[st], &tm_do, &sm.qd_full[st], head * kD, r0);
          if (use_time) tma_load_1d(sm.tq[st], &tm_ts, &sm.qd_full[st], r0 & ~1);
        }
      }
      if (!ok) {  // leave no TMA write in flight into shared memory about to be released
        if (kv_issued > 0) mbar_wait(&sm.kv_full, (kv_issued - 1) & 1, nullptr, nullptr);
        for (int u = gs > kQStages ? gs - kQStages : 0; u < gs; ++u)
          mbar_wait(&sm.qd_full[u % kQStages], (u / kQStages) & 1, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t id_s = idesc_bf16_f32(128, 128, 0, 0);     // S^T, dP^T
      constexpr uint32_t id_kv = idesc_bf16_f32(128, kD, 0, 1);     // dV, dK (B MN-major)
      constexpr uint32_t id_q = idesc_bf16_f32(128, kD, 1, 1);      // dQ (A and B MN-major)
      const uint32_t kb = smem_u32(sm.k), vb = smem_u32(sm.v), dsb = smem_u32(sm.ds);
      int gs = 0, jj = 0;
      bool ok = true;
      for (int w = blockIdx.x; ok && w < total; w += stride, ++jj) {
        const WorkItem it = g.items[nitems - 1 - w / g.H];
        const int kt = it.qtile, L = it.len;
        const int nt = (L + kT - 1) / kT;
        ok = mbar_wait(&sm.kv_full, jj & 1, abort_flag, g.status);
        for (int qt = kt; ok && qt < nt; ++qt, ++gs) {
          const int st = gs % kQStages;
          const bool first = qt == kt;
          ok = mbar_wait(&sm.qd_full[st], (gs / kQStages) & 1, abort_flag, g.status);
          // The previous step's dV, dK and dQ MMAs read P^T / dS^T (aliased with S^T / dP^T)
          // and the dS tile.  This thread issued them before the S^T / dP^T MMAs below, and one
          // thread's MMAs execute in order, so no wait is needed; the epilogue writes the next
          // dS tile only after s_full, whose commit follows those MMAs too.
          if (!ok) break;
          tc_fence_after();
          const uint32_t qb = smem_u32(sm.q[st]), ob = smem_u32(sm.dO[st]);
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            mma_bf16_ss(tmem + kColST, smem_desc_sw128(kb + kk * 32, 16, 1024),
                        smem_desc_sw128(qb + kk * 32, 16, 1024), id_s, kk > 0 ? 1u : 0u);
            mma_bf16_ss(tmem + kColDPT, smem_desc_sw128(vb + kk * 32, 16, 1024),
                        smem_desc_sw128(ob + kk * 32, 16, 1024), id_s, kk > 0 ? 1u : 0u);
          }
          mma_commit(&sm.s_full);
          ok = mbar_wait(&sm.p_full, gs & 1, abort_flag, g.status);
          if (ok && first && jj > 0) ok = mbar_wait(&sm.acc_empty, (jj - 1) & 1, abort_flag, g.status);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk) {  // 16 queries per step; P^T / dS^T columns
            // queries 16 kk..: chunk kk / 2 keeps its 32 queries' pairs in its first 16 columns
            const uint32_t pc = 32 * (kk >> 1) + 8 * (kk & 1);
            mma_bf16_ts(tmem + kColDV, tmem + kColST + pc, smem_desc_sw128(ob + kk * 2048, kTileBytes, 1024),
                        id_kv, (!first || kk > 0) ? 1u : 0u);
            mma_bf16_ts(tmem + kColDK, tmem + kColDPT + pc, smem_desc_sw128(qb + kk * 2048, kTileBytes, 1024),
                        id_kv, (!first || kk > 0) ? 1u : 0u);
          }
          // dQ overwrites the previous step's tile: every epilogue warp drained it before its
          // p_full arrival above
#pragma unroll
          for (int kk = 0; kk < kT / 16; ++kk)  // 16 keys per step
            mma_bf16_ss(tmem + kColDQ, smem_desc_sw128(dsb + kk * 2048, kTileBytes, 1024),
                        smem_desc_sw128(kb + kk * 2048, kTileBytes, 1024), id_q, kk > 0 ? 1u : 0u);
          mma_commit(&sm.qd_empty[st]);
        }
        if (!ok) break;
        mma_commit(&sm.acc_full);
        mma_commit(&sm.kv_empty);
      }
      if (ok && gs > 0) mma_commit(&sm.dq_last);  // the last dQ tile, drained after the loop
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp >= kEpiFirst && warp < kEpiFirst + kEpiWarps) {
    // ---------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int qc = (warp - kEpiFirst) >> 2;  // 32-query chunk of every query tile
    const int hq = qc >> 1, ch = qc & 1;     // its half of the dS tile and place in it
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float alpha = g.alpha;
    // Bias-gradient runs: along one key row the table index changes only where the clamped
    // distance or the time bucket changes, so each thread sums a run in registers and adds it
    // to the shared-memory bin when the index moves on.
    BinRun run_p{-1, 0.f, 1}, run_t{-1, 0.f, 32}, run_t2{-1, 0.f, 32};
    BwdTabs tabs;
    tabs.pos = tab_pos;
    tabs.time = tab_time;
    tabs.bins_pos = bins;
    tabs.bins_time = tbins + lane;
    tabs.alpha = alpha;
    tabs.P = g.P;
    tabs.NB = g.NB;
    tabs.use_pos = use_pos;
    tabs.use_time = use_time;
    // this warp's 32 rows x 16 columns of the dQ tile in TMEM, added to dq_acc at (x, y) by a
    // TMA reduction from this warp's staging rows (64-byte swizzle)
    uint8_t* dq_stage = sm.dqs[warp - kEpiFirst];
    auto drain_dq = [&](int x, int y) {
      uint32_t a[16];
      tmem_ld16(lane_addr + kColDQ + 16 * qc, a);
      tmem_wait_ld16(a);
      if (lane == 0) bulk_wait_read<0>();  // the previous reduction has read the staging rows
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c)
        *reinterpret_cast<uint4*>(dq_stage + stage64_offset(lane, c)) =
            make_uint4(a[4 * c], a[4 * c + 1], a[4 * c + 2], a[4 * c + 3]);
      fence_async_smem();  // read by the TMA (async proxy)
      __syncwarp();
      if (lane == 0) {
        tma_reduce_add_2d(&tm_dq, dq_stage, x, y);
        bulk_commit();
      }
    };
    int dq_x = 0, dq_y = 0;  // where the previous step's dQ tile goes
    int gs = 0, jj = 0;
    bool ok = true;
    for (int w = blockIdx.x; ok && w < total; w += stride, ++jj) {
      const WorkItem it = g.items[nitems - 1 - w / g.H];
      const int head = w % g.H, kt = it.qtile, L = it.len;
      const int n = hist_len(L, g.mask, g.num_candidates);
      const int nt = (L + kT - 1) / kT;
      const int j0 = kt * kT + quad * 32;  // this warp's first key row
      const int jrow = j0 + lane;          // this thread's key row
      const bool jvalid = jrow < L;
      BwdRow row;
      row.jrow = jrow;
      row.jvalid = jvalid;
      row.pj = jrow < n ? jrow : n;
      row.n = n;
      row.L = L;
      row.tj = (use_time && jvalid) ? g.ts[it.row0 + jrow] : 0;
      long long tj_lo = 0, tj_hi = 0;  // the warp's key timestamp range (valid keys)
      if (kFast && use_time) {
        tj_lo = warp_min64(jvalid ? row.tj : LLONG_MAX);
        tj_hi = warp_max64(jvalid ? row.tj : LLONG_MIN);
      }
      for (int qt = kt; ok && qt < nt; ++qt, ++gs) {
        const int st = gs % kQStages;
        ok = warp_wait(&sm.s_full, gs & 1, abort_flag, g.status);
        // the query timestamps came with the Q stage: observe its completion too
        if (ok && use_time) ok = warp_wait(&sm.qd_full[st], (gs / kQStages) & 1, abort_flag, g.status);
        if (!ok) break;
        tc_fence_after();
        // the previous step's dQ (complete: issued before this step's S^T / dP^T)
        if (gs > 0) drain_dq(dq_x, dq_y);
        dq_x = head * kD + 16 * qc;
        dq_y = it.row0 + qt * kT + quad * 32;
        const long long* tq = sm.tq[st] + ((it.row0 + qt * kT) & 1);
        uint8_t* ds_row = sm.ds + hq * kTileBytes + (quad * 32 + lane) * 128;
        const int rr = quad * 32 + lane;
        const uint32_t col = 32 * qc;
        const int i0 = qt * kT + static_cast<int>(col);
        const long long* tq_c = tq + col;
        float cbias = 0.f;
        int cpidx = 0, ctidx = 0;
        const int cls = kFast ? chunk_class(i0, j0, L, n, tabs, tq_c, tj_lo, tj_hi, cbias, cpidx,
                                            ctidx)
                              : kChunkGeneral;
        DiagBins dg{0.f, 0.f};
        const unsigned* tq_lo = reinterpret_cast<const unsigned*>(tq_c);
        const unsigned tj_lo32 = static_cast<unsigned>(row.tj);
#pragma unroll 1
        for (int hf = 0; hf < 2; ++hf) {  // 16 queries at a time (fewer live registers)
          const uint32_t c16 = col + 16 * hf;
          uint32_t pk[8], dk[8];
          if (cls == kChunkZero) {
#pragma unroll
            for (int z = 0; z < 8; ++z) pk[z] = dk[z] = 0u;
          } else {
            uint32_t sv[16], dp[16];
            tmem_ld16(lane_addr + kColST + c16, sv);
            tmem_ld16(lane_addr + kColDPT + c16, dp);
            tmem_wait_ld16(sv);
            tmem_wait_ld16(dp);
            if (cls == kChunkConst)
              bwd_chunk<kChunkConst, 16>(sv, dp, pk, dk, i0 + 16 * hf, tq_c + 16 * hf, row, tabs,
                                         cbias, cpidx, ctidx, run_p, run_t);
            else if (cls == kChunkBandTC)
              bwd_chunk_band<kChunkBandTC, 16>(sv, dp, pk, dk, 16 * hf, i0 + 16 * hf - jrow + g.P, 0,
                                               tq_lo + 32 * hf, tj_lo32, tabs, cbias, ctidx, dg,
                                               run_t, run_t2);
            else if (cls == kChunkBandT32)
              bwd_chunk_band<kChunkBandT32, 16>(sv, dp, pk, dk, 16 * hf, i0 + 16 * hf - jrow + g.P, 0,
                                                tq_lo + 32 * hf, tj_lo32, tabs, cbias, ctidx, dg,
                                                run_t, run_t2);
            else if (cls == kChunkBandT32M)
              bwd_chunk_band<kChunkBandT32, 16, true>(sv, dp, pk, dk, 16 * hf,
                                                      i0 + 16 * hf - jrow + g.P,
                                                      jrow - (i0 + 16 * hf), tq_lo + 32 * hf,
                                                      tj_lo32, tabs, cbias, ctidx, dg, run_t,
                                                      run_t2);
            else if (cls == kChunkBandTH)
              bwd_chunk_band<kChunkBandTH, 16>(sv, dp, pk, dk, 16 * hf, i0 + 16 * hf - jrow + g.P, 0,
                                               tq_lo + 32 * hf, tj_lo32, tabs, cbias, ctidx, dg,
                                               run_t, run_t2);
            else if (cls == kChunkTimeConst)
              bwd_chunk<kChunkTimeConst, 16>(sv, dp, pk, dk, i0 + 16 * hf, tq_c + 16 * hf, row,
                                             tabs, cbias, cpidx, ctidx, run_p, run_t);
            else
              bwd_chunk<kChunkGeneral, 16>(sv, dp, pk, dk, i0 + 16 * hf, tq_c + 16 * hf, row,
                                           tabs, cbias, cpidx, ctidx, run_p, run_t);
          }
          // P^T / (a dS)^T over the chunk's own first 16 columns, already read by this warp
          tmem_st8(lane_addr + kColST + col + 8 * hf, pk);
          tmem_st8(lane_addr + kColDPT + col + 8 * hf, dk);
          // (a dS)^T row to shared memory: 8-query block cb of this half at cb ^ (row & 7)
#pragma unroll
          for (int c2 = 0; c2 < 2; ++c2) {
            const int cb = 4 * ch + 2 * hf + c2;
            const uint4 val = make_uint4(dk[4 * c2], dk[4 * c2 + 1], dk[4 * c2 + 2], dk[4 * c2 + 3]);
            *reinterpret_cast<uint4*>(ds_row + ((cb ^ (rr & 7)) * 16)) = val;
          }
        }
        if (cls >= kChunkBandTC && use_pos)
          dg.flush(tabs.bins_pos, i0 - j0 - 31 + g.P);
        tmem_wait_st();
        fence_async_smem();  // the dS tile is read by the dQ MMA (async proxy)
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.p_full);
      }
      if (!ok) break;
      // the item's dV, dK: this warp's 16 of the 64 columns of each
      ok = warp_wait(&sm.acc_full, jj & 1, abort_flag, g.status);
      if (!ok) break;
      tc_fence_after();
      uint32_t a[16];
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        tmem_ld16(lane_addr + (which ? kColDK : kColDV) + 16 * qc, a);
        tmem_wait_ld16(a);
        if (jvalid) {
          // a layer's backward: dpre = dK (dV) ⊙ SiLU'(Z) before the one rounding to bf16
          const float* zrow = which ? zg.k : zg.v;
          if (zrow != nullptr) {
            zrow += static_cast<int64_t>(it.row0 + jrow) * zg.ld + head * kD + 16 * qc;
#pragma unroll
            for (int e = 0; e < 16; e += 4) {
              const float4 z4 = *reinterpret_cast<const float4*>(zrow + e);
              a[e] = __float_as_uint(__uint_as_float(a[e]) * silu_grad_z(z4.x));
              a[e + 1] = __float_as_uint(__uint_as_float(a[e + 1]) * silu_grad_z(z4.y));
              a[e + 2] = __float_as_uint(__uint_as_float(a[e + 2]) * silu_grad_z(z4.z));
              a[e + 3] = __float_as_uint(__uint_as_float(a[e + 3]) * silu_grad_z(z4.w));
            }
          }
          __nv_bfloat16* dst = (which ? dk_out : dv_out) +
                               static_cast<int64_t>(it.row0 + jrow) * (which ? ld_dk : ld_dv) +
                               head * kD + 16 * qc;
#pragma unroll
          for (int w4 = 0; w4 < 2; ++w4) {
            uint4 vv;
            vv.x = pack_bf16x2(__uint_as_float(a[8 * w4 + 0]), __uint_as_float(a[8 * w4 + 1]));
            vv.y = pack_bf16x2(__uint_as_float(a[8 * w4 + 2]), __uint_as_float(a[8 * w4 + 3]));
            vv.z = pack_bf16x2(__uint_as_float(a[8 * w4 + 4]), __uint_as_float(a[8 * w4 + 5]));
            vv.w = pack_bf16x2(__uint_as_float(a[8 * w4 + 6]), __uint_as_float(a[8 * w4 + 7]));
            reinterpret_cast<uint4*>(dst)[w4] = vv;
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);
    }
    if (ok && gs > 0) {  // the last dQ tile
      ok = warp_wait(&sm.dq_last, 0, abort_flag, g.status);
      if (ok) {
        tc_fence_after();
        drain_dq(dq_x, dq_y);
      }
    }
    if (lane == 0) bulk_wait_all();
    run_p.flush(tabs.bins_pos);
    run_t.flush(tabs.bins_time);
    run_t2.flush(tabs.bins_time);
  }
  tc_fence_before();
  __syncthreads();
  for (int e = threadIdx.x; e < nbins; e += kThreads) {
    float v = 0.f;
    if (e < npos) {
      v = bins[e];
    } else {
      const float* c = tbins + 32 * (e - npos);
#pragma unroll 4
      for (int l = 0; l < 32; ++l) v += c[l];
    }
    if (v != 0.f) atomicAdd(e < npos ? &d_pos[e] : &d_time[e - npos], v);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace
}  // namespace hstu

// ---------------------------------------------------------------------------- host side
namespace hstu {
namespace {
// dQ accumulator (fp32, row stride ld_src) -> bf16 rows; 8 columns per thread (cols and ld_dst
// multiples of 8, dst 16-byte aligned: checked by the caller).
// With z (a layer's backward), the rows are first multiplied by SiLU'(z): dpre of the Q block.
__global__ void f32_to_bf16_rows(const float* __restrict__ src, int64_t ld_src,
                                 __nv_bfloat16* __restrict__ dst, int64_t ld_dst, int rows,
                                 int cols, const float* __restrict__ z, int64_t ld_z) {
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int per_row = cols / 8;
  if (idx >= static_cast<int64_t>(rows) * per_row) return;
  const int64_t r = idx / per_row;
  const int c = static_cast<int>(idx % per_row) * 8;
  float4 a = *reinterpret_cast<const float4*>(src + r * ld_src + c);
  float4 b = *reinterpret_cast<const float4*>(src + r * ld_src + c + 4);
  if (z != nullptr) {
    const float4 za = *reinterpret_cast<const float4*>(z + r * ld_z + c);
    const float4 zb = *reinterpret_cast<const float4*>(z + r * ld_z + c + 4);
    a = make_float4(a.x * silu_grad_z(za.x), a.y * silu_grad_z(za.y), a.z * silu_grad_z(za.z),
                    a.w * silu_grad_z(za.w));
    b = make_float4(b.x * silu_grad_z(zb.x), b.y * silu_grad_z(zb.y), b.z * silu_grad_z(zb.z),
                    b.w * silu_grad_z(zb.w));
  }
  uint4 o;
  o.x = pack_bf16x2(a.x, a.y);
  o.y = pack_bf16x2(a.z, a.w);
  o.z = pack_bf16x2(b.x, b.y);
  o.w = pack_bf16x2(b.z, b.w);
  *reinterpret_cast<uint4*>(dst + r * ld_dst + c) = o;
}
}  // namespace

int attn_bwd_tc_ts_box() { return kTsBox; }

size_t attn_bwd_tc_smem(int P, int NB) {
  return sizeof(BwdSmem) + 1024 + 2 * sizeof(float) * (2 * P + 1 + NB) + 32 * sizeof(float) * NB;
}

// Launches the backward over the work list in g (one 128-row tile per item): tq / tk / tv / tdo
// are 64 x 128 boxes (128-byte swizzle) over Q, K, V, dO; tts a 130-element int64 box over the
// timestamps (used when g.ts and g.rab_time are set); tdq 16 x 32 boxes (64-byte swizzle) over
// dq_acc, fp32 [T, H*64], zeroed here and accumulated by TMA reductions.
// grid: at most one CTA per SM (persistent).  fast: classify each 32 x 32 block of a warp
// (hidden, visible with constant bias terms, visible with a constant time term) and skip the
// per-element work these make unnecessary; otherwise every element takes the per-element path.
// Both give the same P and dS values.  Returns cudaErrorInvalidValue when the bias tables do
// not fit in shared memory.
cudaError_t launch_attn_bwd_tc(const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& tdo,
                               const CUtensorMap& tts, const CUtensorMap& tdq, const AttnGeom& g,
                               __nv_bfloat16* dq, int64_t ld_dq, __nv_bfloat16* dk,
                               int64_t ld_dk, __nv_bfloat16* dv, int64_t ld_dv, float* dq_acc,
                               float* d_pos, float* d_time, int grid, bool fast,
                               const SiluGradZ& zg, cudaStream_t stream) {
  const size_t smem = attn_bwd_tc_smem(g.rab_pos ? g.P : 0, g.rab_time ? g.NB : 0);
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  // d_pos / d_time are accumulated into: the caller zeroes them
  cudaError_t e = cudaMemsetAsync(dq_acc, 0, sizeof(float) * g.T * g.H * 64, stream);
  if (e != cudaSuccess) return e;
  auto kernel = fast ? attn_bwd_tc_kernel<true> : attn_bwd_tc_kernel<false>;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kernel<<<grid, kThreads, smem, stream>>>(tq, tk, tv, tdo, tts, tdq, g, dk, ld_dk, dv, ld_dv,
                                           d_pos, d_time, zg);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t n = static_cast<int64_t>(g.T) * g.H * 8;  // 8 columns per thread
  f32_to_bf16_rows<<<static_cast<int>((n + 255) / 256), 256, 0, stream>>>(
      dq_acc, static_cast<int64_t>(g.H) * 64, dq, ld_dq, g.T, g.H * 64, zg.q, zg.ld);
  return cudaGetLastError();
}
}  // namespace hstu
