// pointwise.cu — HBM-bound and bookkeeping kernels of the HSTU layer:
//   * the jagged work list (device-side validation of seq_offsets + longest-first ordering of
//     the 128-row query tiles, so no host synchronisation is needed),
//   * Norm(AV) ⊙ U — LayerNorm over the H*d_v features of a token, gated elementwise by U
//     ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1 third formula;
//     "HSTU：Scaling Law 的首次探索" §7.1.4, output LayerNorm(A(X)V(X)) ⊙ U(X)),
//   * jagged <-> padded row copies (16-byte vectors, one thread per vector),
//   * the debug export of the log2 time-bucket rule.
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

// ------------------------------------------------------------------------------ work list
// One CTA.  Validates offsets (offsets[0] == 0, offsets[B] == T, every length in [0, max_len]);
// on failure writes the device-check status and an empty list.  An item is a group of
// `group` consecutive 128-row query tiles of one sequence (1 or 2); items are placed in
// decreasing order of cost (KV tiles visited, summed over the group) by a counting sort, so the
// longest items start first.  hist holds max_cost + 1 counters (global workspace).
// cand_only (M-FALCON candidates-only calls): items whose tiles hold no candidate row are left
// out, and every sequence must have at least m tokens.
__device__ __forceinline__ int item_cost(int qt0, int group, int L, int n) {
  int cost = 0;
  for (int a = 0; a < group; ++a) {
    const int qt = qt0 + a;
    if (qt * kTileRows < L) cost += kv_range(qt, L, n).count();
  }
  return cost;
}

// Histogram bins live in shared memory when they fit (the usual case), else in the global
// workspace.  Warps take sequences, lanes take a sequence's items.
constexpr int kWorklistSmemBins = 4096;

__global__ void build_worklist_kernel(const int32_t* __restrict__ offsets, int B, int T,
                                      int max_len, int mask, int m, int group, int cand_only,
                                      WorkItem* __restrict__ items, int32_t* __restrict__ count,
                                      int32_t* __restrict__ hist_global, int max_cost,
                                      int32_t* status) {
  __shared__ int bad;
  __shared__ int hist_smem[kWorklistSmemBins];
  int32_t* hist = max_cost < kWorklistSmemBins ? hist_smem : hist_global;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  if (threadIdx.x == 0) bad = 0;
  for (int c = threadIdx.x; c <= max_cost; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  if (threadIdx.x == 0 && (offsets[0] != 0 || offsets[B] != T)) bad = 1;
  for (int b = threadIdx.x; b < B; b += blockDim.x) {
    const int L = offsets[b + 1] - offsets[b];
    if (L < 0 || L > max_len || (cand_only && L < m)) bad = 1;
  }
  __syncthreads();
  if (bad) {
    if (threadIdx.x == 0) {
      *count = 0;
      atomicExch(status, kStatusDeviceCheck);
    }
    return;
  }
  for (int b = warp; b < B; b += nwarps) {
    const int L = offsets[b + 1] - offsets[b];
    const int n = hist_len(L, mask, m);
    const int nt = (L + kTileRows - 1) / kTileRows;
    for (int qt = lane * group; qt < nt; qt += 32 * group)
      if (!cand_only || (qt + group) * kTileRows > n) atomicAdd(&hist[item_cost(qt, group, L, n)], 1);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive scan in decreasing cost
    int run = 0;
    for (int c = max_cost; c >= 0; --c) {
      const int h = hist[c];
      hist[c] = run;
      run += h;
    }
    *count = run;
  }
  __syncthreads();
  for (int b = warp; b < B; b += nwarps) {
    const int L = offsets[b + 1] - offsets[b];
    const int n = hist_len(L, mask, m);
    const int nt = (L + kTileRows - 1) / kTileRows;
    for (int qt = lane * group; qt < nt; qt += 32 * group) {
      if (cand_only && (qt + group) * kTileRows <= n) continue;
      const int pos = atomicAdd(&hist[item_cost(qt, group, L, n)], 1);
      WorkItem it;
      it.seq = b;
      it.qtile = qt;
      it.row0 = offsets[b];
      it.len = L;
      items[pos] = it;
    }
  }
}

cudaError_t launch_build_worklist(const int32_t* offsets, int B, int T, int max_len, int mask,
                                  int m, int group, int cand_only, WorkItem* items,
                                  int32_t* count, int32_t* hist, int max_cost, int32_t* status,
                                  cudaStream_t stream) {
  build_worklist_kernel<<<1, 1024, 0, stream>>>(offsets, B, T, max_len, mask, m, group, cand_only, items,
                                                count, hist, max_cost, status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------ LayerNorm ⊙ U
template <typename T>
__device__ __forceinline__ float to_f(T v);
template <>
__device__ __forceinline__ float to_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <typename T>
__device__ __forceinline__ T from_f(float v);
template <>
__device__ __forceinline__ float from_f<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }

// One warp per token row; F = H*d_v features, F <= 32 * kMaxPerLane.  Two passes over values
// held in registers: mean, then the biased variance of the centred values (fp32).
constexpr int kMaxPerLane = 32;

template <typename T>
__global__ void ln_gate_kernel(const T* __restrict__ av, int64_t ld_av, const T* __restrict__ u,
                               int64_t ld_u, const float* __restrict__ gamma,
                               const float* __restrict__ beta, float eps, T* __restrict__ g,
                               int64_t ld_g, int rows, int F) {
  const int warp_global = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp_global >= rows) return;
  const T* a = av + static_cast<int64_t>(warp_global) * ld_av;
  const T* uu = u + static_cast<int64_t>(warp_global) * ld_u;
  T* out = g + static_cast<int64_t>(warp_global) * ld_g;
  constexpr int VEC = 16 / sizeof(T);
  float x[kMaxPerLane];
  const bool vec = (F % (32 * VEC) == 0) &&
                   (((reinterpret_cast<uintptr_t>(a) | reinterpret_cast<uintptr_t>(uu) |
                      reinterpret_cast<uintptr_t>(out)) & 15) == 0);
  const int per_lane = F / 32;
  float sum = 0.f;
  if (vec) {
#pragma unroll
    for (int s = 0; s < kMaxPerLane / VEC; ++s) {
      if (s * VEC * 32 >= F) break;
      const uint4 raw = *reinterpret_cast<const uint4*>(a + (s * 32 + lane) * VEC);
      const T* tv = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        x[s * VEC + e] = to_f<T>(tv[e]);
        sum += x[s * VEC + e];
      }
    }
  } else {
    for (int s = 0; s < kMaxPerLane; ++s) {
      const int c = s * 32 + lane;
      x[s] = c < F ? to_f<T>(a[c]) : 0.f;
      sum += x[s];
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float mean = sum / F;
  float sq = 0.f;
  if (vec) {
#pragma unroll
    for (int e = 0; e < kMaxPerLane; ++e)
      if (e < per_lane) {
        const float dlt = x[e] - mean;
        sq += dlt * dlt;
      }
  } else {
    for (int s = 0; s < kMaxPerLane; ++s)
      if (s * 32 + lane < F) {
        const float dlt = x[s] - mean;
        sq += dlt * dlt;
      }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  const float rstd = rsqrtf(sq / F + eps);
  if (vec) {
#pragma unroll
    for (int s = 0; s < kMaxPerLane / VEC; ++s) {
      if (s * VEC * 32 >= F) break;
      const int c0 = (s * 32 + lane) * VEC;
      const uint4 raw = *reinterpret_cast<const uint4*>(uu + c0);
      const T* tu = reinterpret_cast<const T*>(&raw);
      uint4 res;
      T* tr = reinterpret_cast<T*>(&res);
#pragma unroll
      for (int e = 0; e < VEC; ++e) {
        float nv = (x[s * VEC + e] - mean) * rstd;
        if (gamma != nullptr) nv *= gamma[c0 + e];
        if (beta != nullptr) nv += beta[c0 + e];
        tr[e] = from_f<T>(nv * to_f<T>(tu[e]));
      }
      *reinterpret_cast<uint4*>(out + c0) = res;
    }
  } else {
    for (int s = 0; s < kMaxPerLane; ++s) {
      const int c = s * 32 + lane;
      if (c >= F) break;
      float nv = (x[s] - mean) * rstd;
      if (gamma != nullptr) nv *= gamma[c];
      if (beta != nullptr) nv += beta[c];
      out[c] = from_f<T>(nv * to_f<T>(uu[c]));
    }
  }
}

cudaError_t launch_ln_gate(int dtype, const void* av, int64_t ld_av, const void* u, int64_t ld_u,
                           const float* gamma, const float* beta, float eps, void* g,
                           int64_t ld_g, int rows, int F, cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  if (dtype == 0)
    ln_gate_kernel<__nv_bfloat16><<<blocks, threads, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(av), ld_av, static_cast<const __nv_bfloat16*>(u), ld_u,
        gamma, beta, eps, static_cast<__nv_bfloat16*>(g), ld_g, rows, F);
  else
    ln_gate_kernel<float><<<blocks, threads, 0, stream>>>(
        static_cast<const float*>(av), ld_av, static_cast<const float*>(u), ld_u, gamma, beta,
        eps, static_cast<float*>(g), ld_g, rows, F);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ jagged <-> padded copy
// One thread per 16-byte vector of a padded row slot; grid-stride over B * max_len * vecs.
__global__ void jagged_padded_kernel(const int32_t* __restrict__ offsets, int B, int max_len,
                                     uint8_t* __restrict__ jag, int64_t jag_stride,
                                     uint8_t* __restrict__ pad, int64_t pad_stride,
                                     int64_t vecs_per_row, int to_padded) {
  const int64_t total = static_cast<int64_t>(B) * max_len * vecs_per_row;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t v = idx % vecs_per_row;
    const int64_t slot = idx / vecs_per_row;
    const int b = static_cast<int>(slot / max_len);
    const int r = static_cast<int>(slot % max_len);
    const int s = offsets[b];
    const int L = offsets[b + 1] - s;
    uint4* pdst = reinterpret_cast<uint4*>(pad + slot * pad_stride) + v;
    if (to_padded) {
      uint4 val = make_uint4(0, 0, 0, 0);
      if (r < L) val = reinterpret_cast<const uint4*>(jag + static_cast<int64_t>(s + r) * jag_stride)[v];
      *pdst = val;
    } else if (r < L) {
      reinterpret_cast<uint4*>(jag + static_cast<int64_t>(s + r) * jag_stride)[v] = *pdst;
    }
  }
}

cudaError_t launch_jagged_padded(const int32_t* offsets, int B, int max_len, const void* jag,
                                 int64_t jag_stride, void* pad, int64_t pad_stride,
                                 int64_t row_bytes, int to_padded, int num_sms,
                                 cudaStream_t stream) {
  const int64_t total = static_cast<int64_t>(B) * max_len * (row_bytes / 16);
  if (total <= 0) return cudaSuccess;
  int64_t blocks = (total + 255) / 256;
  const int64_t cap = static_cast<int64_t>(num_sms) * 8;
  if (blocks > cap) blocks = cap;
  jagged_padded_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(
      offsets, B, max_len, static_cast<uint8_t*>(const_cast<void*>(jag)), jag_stride,
      static_cast<uint8_t*>(pad), pad_stride, row_bytes / 16, to_padded);
  return cudaGetLastError();
}

// ------------------------------------------------------------------- bounded-wait probe
// One mbarrier whose phase nothing completes, waited on with the bounded wait every kernel of
// the library uses: the wait gives up after its limit, writes the timeout code into the status
// word and the kernel returns, so the failure reaches the host and the context stays usable.
__global__ void wait_timeout_probe_kernel(int32_t* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, status);
}

cudaError_t launch_wait_timeout_probe(int32_t* status, cudaStream_t stream) {
  wait_timeout_probe_kernel<<<1, 32, 0, stream>>>(status);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------- time buckets
__global__ void time_bucket_kernel(const int64_t* __restrict__ dt, int n, int32_t* __restrict__ out,
                                   int nb) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = time_bucket64(dt[i], nb);
}

cudaError_t launch_time_buckets(const int64_t* dt, int n, int32_t* out, int nb,
                                cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  time_bucket_kernel<<<(n + 255) / 256, 256, 0, stream>>>(dt, n, out, nb);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ bias-index rules (debug)
// One thread per query; each rule calls the bias_index.cuh function the attention kernels call
// at that point, so the output is what the kernels compute.  Rules and inputs: see
// hstu_debug_bias_index() in include/hstu.h.
__global__ void bias_index_kernel(int rule, const int64_t* __restrict__ in, int n, int param,
                                  int32_t* __restrict__ out) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  int r = -1;
  switch (rule) {
    case 0: r = time_bucket64(in[i], param); break;
    case 1: r = bucket_small(static_cast<int>(in[i]), param - 1); break;
    case 2: r = time_table_src(log2_small(static_cast<int>(in[i])), param); break;
    case 3: r = bucket32(static_cast<int>(in[i]), param - 1); break;
    case 4: {  // (dt_lo, dt_hi, dt): the two-bucket choice, -1 if the row spans more buckets
      const int b_lo = bucket_small(static_cast<int>(in[3 * i]), param - 1);
      const int b_hi = bucket_small(static_cast<int>(in[3 * i + 1]), param - 1);
      if (b_hi <= b_lo + 1)
        r = threshold_takes_hi(static_cast<int>(in[3 * i + 2]), threshold_of(b_lo)) ? b_hi : b_lo;
      break;
    }
    case 5: {  // (p_i, j, -): lane (j mod 4) of the shifted table's entry for key j
      const int p_i = static_cast<int>(in[3 * i]), j = static_cast<int>(in[3 * i + 1]);
      const int c0t = j - j % kPairKvRows;         // first key of j's tile
      const int c = (j - c0t) & ~3;                // the 4-aligned column of the load
      const int x = pos4_row(p_i + param - c0t, c, 2 * param);
      r = pos4_lane_src(x, j - c0t - c, 2 * param);
      break;
    }
    case 6: {  // (p_i, j, n): candidate segments, key position min(j, n), lane 0
      const int x = pos4_general_row(static_cast<int>(in[3 * i]) + param,
                                     static_cast<int>(in[3 * i + 1]),
                                     static_cast<int>(in[3 * i + 2]), 2 * param);
      r = pos4_lane_src(x, 0, 2 * param);
      break;
    }
    case 7:  // (p_min, j_last, -): 2P when the segment's position term is constant, else -1
      r = pos_segment_beyond_clamp(static_cast<int>(in[3 * i]), static_cast<int>(in[3 * i + 1]),
                                   param)
              ? pos4_lane_src(2 * param + 3, 0, 2 * param)
              : -1;
      break;
    case 8:  // (p_i, p_j, -): the direct clamp
      r = pos_index_direct(static_cast<int>(in[3 * i]), static_cast<int>(in[3 * i + 1]), param);
      break;
    default: break;
  }
  out[i] = r;
}

cudaError_t launch_bias_index(int rule, const int64_t* in, int n, int param, int32_t* out,
                              cudaStream_t stream) {
  if (n <= 0) return cudaSuccess;
  bias_index_kernel<<<(n + 255) / 256, 256, 0, stream>>>(rule, in, n, param, out);
  return cudaGetLastError();
}

}  // namespace hstu
