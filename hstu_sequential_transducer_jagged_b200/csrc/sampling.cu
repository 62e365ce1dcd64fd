// sampling.cu — Stochastic Length ("HSTU：Scaling Law 的首次探索" §7.1.5): during training a long
// user sequence is, at random, replaced by a shorter subsequence of its tokens, which cuts the
// O(n²) attention work.  Reading of the page's garbled formula (the library's convention):
//   a sequence of n tokens stays whole when n <= N^{α/2}; otherwise, with probability
//   1 - N^α / n², it becomes the sub_len = floor(N^{α/2}) tokens with the smallest random keys
//   (ties to the lower index), kept in their order; otherwise it stays whole.
// The random draws are inputs (u[b] per sequence, key[t] per token), so the result is a pure
// function of them.  Then the jagged offsets are rebuilt and the kept tokens' indices listed;
// hstu_gather_rows moves any per-token array into the new layout.
//
// Kernels: one CTA per sequence selects its tokens (a radix select of the sub_len-th smallest
// key over 32 bit steps, then two block scans in index order), one CTA scans the new lengths
// into offsets, and one CTA per sequence writes its kept indices at their new place.
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kSelThreads = 1024;

// Block-wide sum of an int (every thread gets the total).  red: shared [32].
__device__ __forceinline__ int block_sum(int v, int* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = __reduce_add_sync(0xffffffffu, v);
  __syncthreads();  // red is free
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int t = lane < static_cast<int>(blockDim.x >> 5) ? red[lane] : 0;
  t = __reduce_add_sync(0xffffffffu, t);
  return t;
}

// Exclusive block scan of a 0/1 flag in thread order; *total gets the block's count.
// red: shared [32].
__device__ __forceinline__ int block_excl_scan(bool flag, int* red, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, flag);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  __syncthreads();  // red is free
  if (lane == 0) red[warp] = __popc(bal);
  __syncthreads();
  int before = 0, all = 0;
  const int nw = static_cast<int>(blockDim.x >> 5);
  for (int w = 0; w < nw; ++w) {
    const int c = red[w];
    before += w < warp ? c : 0;
    all += c;
  }
  *total = all;
  return before + in_warp;
}

__global__ void __launch_bounds__(kSelThreads)
    stoch_select_kernel(const int32_t* __restrict__ off, int B, int T, int max_len, int sub_len,
                        double n_alpha, const float* __restrict__ u,
                        const uint32_t* __restrict__ keys, int32_t* __restrict__ local_idx,
                        int32_t* __restrict__ lens, int32_t* status) {
  __shared__ int red[32];
  const int b = blockIdx.x;
  const int s = off[b];
  int n = off[b + 1] - s;
  const bool bad = n < 0 || n > max_len || s < 0 || s + n > T || (b == 0 && s != 0) ||
                   (b == B - 1 && off[B] != T);
  if (bad) {
    if (threadIdx.x == 0) {
      atomicExch(status, kStatusDeviceCheck);
      lens[b] = 0;
    }
    return;
  }
  const double nd = static_cast<double>(n);
  const bool sub = n > sub_len && static_cast<double>(u[b]) < 1.0 - n_alpha / (nd * nd);
  if (!sub) {
    for (int r = threadIdx.x; r < n; r += blockDim.x) local_idx[s + r] = r;
    if (threadIdx.x == 0) lens[b] = n;
    return;
  }
  // theta = the largest value with fewer than sub_len keys below it: the sub_len-th smallest key
  uint32_t prefix = 0;
  int c_less = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t t = prefix | (1u << bit);
    int c = 0;
    for (int r = threadIdx.x; r < n; r += blockDim.x) c += keys[s + r] < t ? 1 : 0;
    c = block_sum(c, red);
    if (c < sub_len) {
      prefix = t;
      c_less = c;
    }
  }
  // (if no step kept its bit, theta = 0 and no key lies below it)
  const uint32_t theta = prefix;
  const int need_eq = sub_len - c_less;  // keys equal to theta taken, lowest indices first
  int run_eq = 0, run_sel = 0;
  for (int base = 0; base < n; base += blockDim.x) {
    const int r = base + threadIdx.x;
    const uint32_t k = r < n ? keys[s + r] : 0u;
    const bool is_less = r < n && k < theta;
    const bool is_eq = r < n && k == theta;
    int tot_eq = 0, tot_sel = 0;
    const int eq_rank = run_eq + block_excl_scan(is_eq, red, &tot_eq);
    const bool sel = is_less || (is_eq && eq_rank < need_eq);
    const int pos = run_sel + block_excl_scan(sel, red, &tot_sel);
    if (sel) local_idx[s + pos] = r;
    run_eq += tot_eq;
    run_sel += tot_sel;
  }
  if (threadIdx.x == 0) lens[b] = sub_len;
}

// new_off[0] = 0, new_off[b + 1] = new_off[b] + lens[b]; one CTA, in chunks of its threads.
__global__ void __launch_bounds__(kSelThreads)
    offsets_scan_kernel(const int32_t* __restrict__ lens, int B, int32_t* __restrict__ new_off) {
  __shared__ int red[32];
  __shared__ int carry;
  if (threadIdx.x == 0) {
    carry = 0;
    new_off[0] = 0;
  }
  __syncthreads();
  for (int base = 0; base < B; base += blockDim.x) {
    const int b = base + threadIdx.x;
    const int v = b < B ? lens[b] : 0;
    // inclusive scan of v within the chunk: warp scan, then the warps' totals
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    __syncthreads();
    if (lane == 31) red[warp] = x;
    __syncthreads();
    int before = 0, all = 0;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
      before += w < warp ? red[w] : 0;
      all += red[w];
    }
    const int c0 = carry;
    if (b < B) new_off[b + 1] = c0 + before + x;
    __syncthreads();
    if (threadIdx.x == 0) carry = c0 + all;
    __syncthreads();
  }
}

// kept[new_off[b] + r] = off[b] + local_idx[off[b] + r] for r < lens[b].
__global__ void kept_scatter_kernel(const int32_t* __restrict__ off,
                                    const int32_t* __restrict__ new_off,
                                    const int32_t* __restrict__ lens,
                                    const int32_t* __restrict__ local_idx,
                                    int32_t* __restrict__ kept) {
  const int b = blockIdx.x;
  const int s = off[b], d = new_off[b], n = lens[b];
  for (int r = threadIdx.x; r < n; r += blockDim.x) kept[d + r] = s + local_idx[s + r];
}

// dst row r = src row index[r] for r < min(*count, n) (count NULL: n rows); V-byte vectors.
template <typename Vec>
__global__ void gather_rows_kernel(const uint8_t* __restrict__ src, int64_t src_stride,
                                   const int32_t* __restrict__ index, const int32_t* count, int n,
                                   uint8_t* __restrict__ dst, int64_t dst_stride,
                                   int64_t vecs_per_row) {
  const int rows = count != nullptr ? min(*count, n) : n;
  const int64_t total = static_cast<int64_t>(rows) * vecs_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vecs_per_row, v = i % vecs_per_row;
    const int64_t from = index[r];
    reinterpret_cast<Vec*>(dst + r * dst_stride)[v] =
        reinterpret_cast<const Vec*>(src + from * src_stride)[v];
  }
}

// dst row index[r] = src row r for r < n; V-byte vectors.
template <typename Vec>
__global__ void scatter_rows_kernel(const uint8_t* __restrict__ src, int64_t src_stride,
                                    const int32_t* __restrict__ index, int n,
                                    uint8_t* __restrict__ dst, int64_t dst_stride,
                                    int64_t vecs_per_row) {
  const int64_t total = static_cast<int64_t>(n) * vecs_per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / vecs_per_row, v = i % vecs_per_row;
    const int64_t to = index[r];
    reinterpret_cast<Vec*>(dst + to * dst_stride)[v] =
        reinterpret_cast<const Vec*>(src + r * src_stride)[v];
  }
}

// M-FALCON candidate rows: idx[b m + c] = offsets[b + 1] - m + c, the c-th of the last m tokens of
// sequence b.  A sequence shorter than m sets the device-check status (its rows point at row 0).
__global__ void candidate_rows_kernel(const int32_t* __restrict__ off, int B, int m,
                                      int32_t* __restrict__ idx, int32_t* status) {
  const int64_t total = static_cast<int64_t>(B) * m;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(i / m), c = static_cast<int>(i % m);
    const int s = off[b], e = off[b + 1];
    if (e - s < m) {
      atomicExch(status, kStatusDeviceCheck);
      idx[i] = 0;
    } else {
      idx[i] = e - m + c;
    }
  }
}

}  // namespace

cudaError_t launch_candidate_rows(const int32_t* off, int B, int m, int32_t* idx, int32_t* status,
                                  cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(B) * m;
  if (total <= 0) return cudaSuccess;
  const int64_t blocks = (total + 255) / 256;
  candidate_rows_kernel<<<static_cast<int>(blocks < 4096 ? blocks : 4096), 256, 0, stream>>>(
      off, B, m, idx, status);
  return cudaGetLastError();
}

cudaError_t launch_scatter_rows(const void* src, int64_t src_stride, const int32_t* index, int n,
                                void* dst, int64_t dst_stride, int64_t row_bytes, int num_sms,
                                cudaStream_t stream) {
  if (n <= 0 || row_bytes <= 0) return cudaSuccess;
  const uintptr_t align = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                          static_cast<uintptr_t>(src_stride) |
                          static_cast<uintptr_t>(dst_stride) | static_cast<uintptr_t>(row_bytes);
  const int vb = (align % 16 == 0) ? 16 : (align % 8 == 0) ? 8 : 4;
  const int64_t vecs = row_bytes / vb;
  const int64_t total = static_cast<int64_t>(n) * vecs;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
  const auto* s = static_cast<const uint8_t*>(src);
  auto* d = static_cast<uint8_t*>(dst);
  if (vb == 16)
    scatter_rows_kernel<uint4><<<static_cast<int>(blocks), 256, 0, stream>>>(
        s, src_stride, index, n, d, dst_stride, vecs);
  else if (vb == 8)
    scatter_rows_kernel<uint2><<<static_cast<int>(blocks), 256, 0, stream>>>(
        s, src_stride, index, n, d, dst_stride, vecs);
  else
    scatter_rows_kernel<uint32_t><<<static_cast<int>(blocks), 256, 0, stream>>>(
        s, src_stride, index, n, d, dst_stride, vecs);
  return cudaGetLastError();
}

cudaError_t launch_stochastic_length(const int32_t* off, int B, int T, int max_len, int sub_len,
                                     double n_alpha, const float* u, const uint32_t* keys,
                                     int32_t* local_idx, int32_t* lens, int32_t* new_off,
                                     int32_t* kept, int32_t* status, cudaStream_t stream) {
  if (B <= 0) return cudaMemsetAsync(new_off, 0, sizeof(int32_t), stream);
  stoch_select_kernel<<<B, kSelThreads, 0, stream>>>(off, B, T, max_len, sub_len, n_alpha, u,
                                                      keys, local_idx, lens, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  offsets_scan_kernel<<<1, kSelThreads, 0, stream>>>(lens, B, new_off);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  kept_scatter_kernel<<<B, 256, 0, stream>>>(off, new_off, lens, local_idx, kept);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, int64_t src_stride, const int32_t* index,
                               const int32_t* count, int n, void* dst, int64_t dst_stride,
                               int64_t row_bytes, int num_sms, cudaStream_t stream) {
  if (n <= 0 || row_bytes <= 0) return cudaSuccess;
  const uintptr_t align = reinterpret_cast<uintptr_t>(src) | reinterpret_cast<uintptr_t>(dst) |
                          static_cast<uintptr_t>(src_stride) |
                          static_cast<uintptr_t>(dst_stride) | static_cast<uintptr_t>(row_bytes);
  const int vb = (align % 16 == 0) ? 16 : (align % 8 == 0) ? 8 : 4;
  const int64_t vecs = row_bytes / vb;
  const int64_t total = static_cast<int64_t>(n) * vecs;
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
  const auto* s = static_cast<const uint8_t*>(src);
  auto* d = static_cast<uint8_t*>(dst);
  if (vb == 16)
    gather_rows_kernel<uint4><<<static_cast<int>(blocks), 256, 0, stream>>>(
        s, src_stride, index, count, n, d, dst_stride, vecs);
  else if (vb == 8)
    gather_rows_kernel<uint2><<<static_cast<int>(blocks), 256, 0, stream>>>(
        s, src_stride, index, count, n, d, dst_stride, vecs);
  else
    gather_rows_kernel<uint32_t><<<static_cast<int>(blocks), 256, 0, stream>>>(
        s, src_stride, index, count, n, d, dst_stride, vecs);
  return cudaGetLastError();
}

}  // namespace hstu
