// bias_index.cuh — the integer rules that turn a (query, key) pair into indices of the relative
// bias tables, exactly as the attention kernels evaluate them.
//
//   rab_{p,t}(i, j) = rab_pos[clamp(p_i - p_j, -P, P) + P] + rab_time[bucket(t_i - t_j)],
//   bucket(dt) = clamp(floor(log2(max(1, dt))), 0, NB - 1)
// ("HSTU：Scaling Law 的首次探索" §7.1.4 innovation 2: a bias from the position and time
// differences; the log2 time buckets and the position clamp are the readings this library fixes).
//
// The kernels never materialise these indices; they fold them into the epilogue in several
// forms (the 64-bit bucket, a bucket from the fp32 exponent for differences below 2^23, a
// count-leading-zeros bucket on 32-bit differences, a two-bucket threshold, and a 4-wide shifted
// copy of the position table).  Every one of those forms lives here, and both the attention
// kernels and the debug export hstu_debug_bias_index() call these same functions, so the export
// shows bit for bit what the kernels compute.
#pragma once
#include <stdint.h>

namespace hstu {

// Rows of a key/value tile of the paired head-width-64 forward kernel; the 4-wide shifted
// position table is indexed relative to the tile's first key.
constexpr int kPairKvRows = 96;

// Entries of the half-scaled time table the forward kernels keep in shared memory.  No bucket
// exceeds 62 (floor(log2) of a positive int64), so 64 entries hold every index.
constexpr int kTimeTableEntries = 64;

__host__ __device__ __forceinline__ int clampi(int x, int lo, int hi) {
  return x < lo ? lo : (x > hi ? hi : x);
}

// ------------------------------------------------------------------------------- time buckets
// floor(log2(max(1, dt))) clamped to [0, nb-1], exactly, on the 64-bit difference (count of
// leading zeros).
__device__ __forceinline__ int time_bucket64(long long dt, int nb) {
  unsigned long long d = dt < 1 ? 1ull : static_cast<unsigned long long>(dt);
  int b = 63 - __clzll(static_cast<long long>(d));
  return b < nb - 1 ? b : nb - 1;
}

// floor(log2(max(1, d))) for d < 2^23 without a count-leading-zeros: 2^23 + d is exact in fp32,
// so after subtracting 2^23 the biased exponent of the difference is 127 + the bit length of d
// minus one.  d is clamped to [1, 2^23 - 1] first (the kernels use it only inside that range).
__device__ __forceinline__ int log2_small(int d) {
  d = d < 1 ? 1 : (d > 0x7FFFFF ? 0x7FFFFF : d);
  const float f = __int_as_float(0x4B000000 | d) - 8388608.0f;
  return (__float_as_int(f) >> 23) - 127;
}

// The bucket of a difference below 2^23, clamped to nbm1 = NB - 1 (per-row bucket bounds).
__device__ __forceinline__ int bucket_small(int d, int nbm1) {
  const int b = log2_small(d);
  return b < nbm1 ? b : nbm1;
}

// The bucket of a 32-bit difference (|d| < 2^31), clamped to nbm1, by counting leading zeros
// (the forward kernel's tile classifier, on timestamps taken relative to a nearby reference).
__device__ __forceinline__ int bucket32(int d, int nbm1) {
  const int b = d < 1 ? 0 : 31 - __clz(d);
  return b < nbm1 ? b : nbm1;
}

// Entry e of the kernels' time table holds rab_time[time_table_src(e, NB)]: indices past the
// last bucket read the last bucket, which is the clamp to NB - 1.
__host__ __device__ __forceinline__ int time_table_src(int e, int nb) { return e < nb ? e : nb - 1; }

// Two-bucket rows: when every key of a row segment lies in bucket b_lo or b_hi <= b_lo + 1, the
// kernel picks b_hi for a difference d >= 2^(b_lo + 1) and b_lo otherwise.
__device__ __forceinline__ int threshold_of(int b_lo) { return 1 << (b_lo + 1); }
__device__ __forceinline__ bool threshold_takes_hi(int d, int thr) { return d >= thr; }

// ---------------------------------------------------------------------------- position index
// The direct form: clamp(p_i - p_j, -P, P) + P.
__device__ __forceinline__ int pos_index_direct(int p_i, int p_j, int P) {
  return clampi(p_i - p_j, -P, P) + P;
}

// The 4-wide shifted table of the paired forward kernel: entry x holds the table values at
// pos4_lane_src(x, u, 2P) for u = 0..3, so one 16-byte load gives the bias of four consecutive
// keys.  For a query at position p_i and a tile starting at key c0t, pbase = p_i + P - c0t, and
// the keys c0t + c + u (c a multiple of 4) read lane u of entry pos4_row(pbase, c, 2P).  Both
// clamps are exact: past either end of the band every lane reads the table's first or last
// entry.
__device__ __forceinline__ int pos4_row(int pbase, int c, int P2) { return clampi(pbase - c, 0, P2 + 3); }
__device__ __forceinline__ int pos4_lane_src(int x, int u, int P2) { return clampi(x - u, 0, P2); }

// M-FALCON segments (candidate rows meeting candidate keys): the key's position is min(j, n)
// and lane 0 of entry clamp(p_i + P - min(j, n), 0, 2P) is read.
__device__ __forceinline__ int pos4_general_row(int pi_plus_p, int j, int n, int P2) {
  return clampi(pi_plus_p - (j < n ? j : n), 0, P2);
}

// A row segment whose smallest query position is p_min and whose last key is j_last takes one
// constant position term (the table's last entry, index 2P) iff p_min - j_last >= P.
__device__ __forceinline__ bool pos_segment_beyond_clamp(int p_min, int j_last, int P) {
  return !(p_min - j_last < P);
}

}  // namespace hstu
