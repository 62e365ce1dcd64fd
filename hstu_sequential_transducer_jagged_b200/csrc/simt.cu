// simt.cu — CUDA-core kernels of the HSTU layer for the fp32 data type and for head widths the
// tensor-core kernels do not take, plus the attention backward:
//   * attention forward: one thread per query row of a 128-row tile, keys/values staged through
//     shared memory 32 rows at a time, fp32 accumulation;
//   * GEMM with the SiLU or residual epilogue (64x64 output tiles, 4x4 per thread);
//   * attention backward (three kernels, each recomputing the scores S = alpha QKᵀ + rab):
//     dQ (+ the bias-table gradients, reduced per CTA in shared memory, one global atomic per
//     table entry per CTA), dK, dV.
// Formulas: "万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1; the bias gradient is the
// N×N rab backward that "6.2 HSTU的工程突破" §6.2.3 names as the RAB's cost.
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

template <typename T>
__device__ __forceinline__ float ld_f(const T* p);
template <>
__device__ __forceinline__ float ld_f<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float ld_f<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T>
__device__ __forceinline__ void st_f(T* p, float v);
template <>
__device__ __forceinline__ void st_f<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void st_f<__nv_bfloat16>(__nv_bfloat16* p, float v) { *p = __float2bfloat16_rn(v); }

__device__ __forceinline__ float silu_f(float x) { return x / (1.0f + expf(-x)); }
__device__ __forceinline__ float silu_grad_f(float x) {
  const float s = 1.0f / (1.0f + expf(-x));
  return s * (1.0f + x * (1.0f - s));
}

constexpr int kKvChunk = 32;

// Bias of the pair (i, j) (indices local to the sequence) and the two table indices.
struct PairBias {
  float value;
  int pidx;
  int tidx;
  int yidx;  // token-type pair index, -1 without the type term
};

// row0: the sequence's first token (for the token types).
__device__ __forceinline__ PairBias pair_bias(const AttnGeom& g, int i, int j, int n, long long ti,
                                              long long tj, int row0) {
  PairBias b{0.f, -1, -1, -1};
  if (g.rab_type != nullptr) {
    b.yidx = g.types[row0 + i] * g.NT + g.types[row0 + j];
    b.value += g.rab_type[b.yidx];
  }
  if (g.rab_pos != nullptr) {
    const int pi = i < n ? i : n;
    const int pj = j < n ? j : n;
    b.pidx = pos_index_direct(pi, pj, g.P);
    b.value += g.rab_pos[b.pidx];
  }
  if (g.ts != nullptr && g.rab_time != nullptr) {
    b.tidx = time_bucket64(ti - tj, g.NB);
    b.value += g.rab_time[b.tidx];
  }
  return b;
}

__device__ __forceinline__ bool visible(int i, int j, int n) { return j <= i && (j < n || j == i); }

}  // namespace

// ------------------------------------------------------------------------ forward (SIMT)
template <typename T, int D>
__global__ void __launch_bounds__(128)
    attn_fwd_simt_kernel(AttnGeom g, const T* __restrict__ q, int64_t ld_q,
                         const T* __restrict__ k, int64_t ld_k, const T* __restrict__ v,
                         int64_t ld_v, T* __restrict__ o, int64_t ld_o) {
  const int item_idx = blockIdx.x / g.H;
  const int h = blockIdx.x % g.H;
  if (item_idx >= *g.item_count) return;
  const WorkItem it = g.items[item_idx];
  __shared__ float ks[kKvChunk][D];
  __shared__ float vs[kKvChunk][D];
  __shared__ long long tss[kKvChunk];
  const int L = it.len;
  const int n = hist_len(L, g.mask, g.num_candidates);
  const int i = it.qtile * kTileRows + threadIdx.x;
  const bool valid = i < L;
  float qr[D];
  float acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    qr[d] = valid ? ld_f<T>(q + static_cast<int64_t>(it.row0 + i) * ld_q + h * D + d) : 0.f;
    acc[d] = 0.f;
  }
  const long long ti = (valid && g.ts != nullptr) ? g.ts[it.row0 + i] : 0;
  const KvRange kr = kv_range(it.qtile, L, n);
  for (int t = 0; t < kr.count(); ++t) {
    const int c0 = kr.tile(t, it.qtile) * kTileRows;
    for (int cc = 0; cc < kTileRows; cc += kKvChunk) {
      __syncthreads();
      for (int e = threadIdx.x; e < kKvChunk * D; e += blockDim.x) {
        const int r = e / D, d = e % D;
        const int j = c0 + cc + r;
        const bool in = j < L;
        ks[r][d] = in ? ld_f<T>(k + static_cast<int64_t>(it.row0 + j) * ld_k + h * D + d) : 0.f;
        vs[r][d] = in ? ld_f<T>(v + static_cast<int64_t>(it.row0 + j) * ld_v + h * D + d) : 0.f;
      }
      if (threadIdx.x < kKvChunk) {
        const int j = c0 + cc + threadIdx.x;
        tss[threadIdx.x] = (g.ts != nullptr && j < L) ? g.ts[it.row0 + j] : 0;
      }
      __syncthreads();
      if (!valid) continue;
      for (int r = 0; r < kKvChunk; ++r) {
        const int j = c0 + cc + r;
        if (j >= L || !visible(i, j, n)) continue;
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < D; ++d) s = fmaf(qr[d], ks[r][d], s);
        const PairBias pb = pair_bias(g, i, j, n, ti, tss[r], it.row0);
        const float p = silu_f(g.alpha * s + pb.value);
#pragma unroll
        for (int d = 0; d < D; ++d) acc[d] = fmaf(p, vs[r][d], acc[d]);
      }
    }
  }
  if (valid) {
#pragma unroll
    for (int d = 0; d < D; ++d) st_f<T>(o + static_cast<int64_t>(it.row0 + i) * ld_o + h * D + d, acc[d]);
  }
}

// --------------------------------------------------------------------------- GEMM (SIMT)
// C[M,N] = epi(A[M,K] B[K,N] + bias): EPI 0 SiLU, EPI 1 + residual R[M,N].
template <typename T, int EPI>
__global__ void __launch_bounds__(256)
    gemm_simt_kernel(const T* __restrict__ A, int64_t lda, const T* __restrict__ B, int64_t ldb,
                     int M, int N, int K, const float* __restrict__ bias,
                     const T* __restrict__ R, int64_t ldr, T* __restrict__ C, int64_t ldc) {
  __shared__ float as[16][64 + 1];
  __shared__ float bs[16][64 + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e / 64, mm = e % 64;
      const int gm = m0 + mm, gk = k0 + kk;
      as[kk][mm] = (gm < M && gk < K) ? ld_f<T>(A + static_cast<int64_t>(gm) * lda + gk) : 0.f;
      const int gn = n0 + mm;
      bs[kk][mm] = (gn < N && gk < K) ? ld_f<T>(B + static_cast<int64_t>(gk) * ldb + gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(as[kk][ty * 4 + a], bs[kk][tx * 4 + b], acc[a][b]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int gm = m0 + ty * 4 + a;
    if (gm >= M) continue;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int gn = n0 + tx * 4 + b;
      if (gn >= N) continue;
      float x = acc[a][b] + (bias != nullptr ? bias[gn] : 0.f);
      if (EPI == 0) x = silu_f(x);
      else x += ld_f<T>(R + static_cast<int64_t>(gm) * ldr + gn);
      st_f<T>(C + static_cast<int64_t>(gm) * ldc + gn, x);
    }
  }
}

// ----------------------------------------------------------------------- backward (SIMT)
// KIND 0: dQ_i = alpha Σ_j dS_ij K_j, plus the bias-table gradients (thread = query row i).
// KIND 1: dK_j = alpha Σ_i dS_ij Q_i (thread = key row j).
// KIND 2: dV_j = Σ_i A_ij dO_i (thread = key row j).
// dS_ij = (dO_i · V_j) SiLU'(S_ij) on visible pairs.
template <typename T, int D, int KIND>
__global__ void __launch_bounds__(128)
    attn_bwd_simt_kernel(AttnGeom g, const T* __restrict__ q, int64_t ld_q,
                         const T* __restrict__ k, int64_t ld_k, const T* __restrict__ v,
                         int64_t ld_v, const T* __restrict__ d_o, int64_t ld_do,
                         T* __restrict__ out, int64_t ld_out, float* __restrict__ d_pos,
                         float* __restrict__ d_time) {
  const int item_idx = blockIdx.x / g.H;
  const int h = blockIdx.x % g.H;
  if (item_idx >= *g.item_count) return;
  const WorkItem it = g.items[item_idx];
  const int L = it.len;
  const int n = hist_len(L, g.mask, g.num_candidates);
  // the thread's own row: a query row (KIND 0) or a key row (KIND 1, 2)
  const int r = it.qtile * kTileRows + threadIdx.x;
  const bool valid = r < L;
  const int64_t grow = it.row0 + r;
  __shared__ float xs[kKvChunk][D];   // partner rows: K (KIND 0) or Q (KIND 1, 2)
  __shared__ float ys[kKvChunk][D];   // partner rows: V (KIND 0) or dO (KIND 1, 2)
  __shared__ long long tss[kKvChunk];
  extern __shared__ float bias_grad[];  // KIND 0: [2P+1] position, [NB] time, [NT^2] type
  const int npos = (g.rab_pos != nullptr) ? 2 * g.P + 1 : 0;
  const int ntime = (g.ts != nullptr && g.rab_time != nullptr) ? g.NB : 0;
  const int ntype = (g.rab_type != nullptr) ? g.NT * g.NT : 0;
  if (KIND == 0) {
    for (int e = threadIdx.x; e < npos + ntime + ntype; e += blockDim.x) bias_grad[e] = 0.f;
  }
  float a[D], b[D], acc[D];
#pragma unroll
  for (int d = 0; d < D; ++d) {
    if (KIND == 0) {
      a[d] = valid ? ld_f<T>(q + grow * ld_q + h * D + d) : 0.f;
      b[d] = valid ? ld_f<T>(d_o + grow * ld_do + h * D + d) : 0.f;
    } else {
      a[d] = valid ? ld_f<T>(k + grow * ld_k + h * D + d) : 0.f;
      b[d] = valid ? ld_f<T>(v + grow * ld_v + h * D + d) : 0.f;
    }
    acc[d] = 0.f;
  }
  const long long tr = (valid && g.ts != nullptr) ? g.ts[grow] : 0;
  // partner range: keys 0 .. (tile end) for KIND 0; queries from this tile's start to L for 1, 2
  const int p_begin = (KIND == 0) ? 0 : it.qtile * kTileRows;
  const int p_end = (KIND == 0) ? min(L, (it.qtile + 1) * kTileRows) : L;
  for (int c0 = p_begin; c0 < p_end; c0 += kKvChunk) {
    __syncthreads();
    for (int e = threadIdx.x; e < kKvChunk * D; e += blockDim.x) {
      const int rr = e / D, d = e % D;
      const int j = c0 + rr;
      const bool in = j < p_end;
      const int64_t gj = it.row0 + j;
      if (KIND == 0) {
        xs[rr][d] = in ? ld_f<T>(k + gj * ld_k + h * D + d) : 0.f;
        ys[rr][d] = in ? ld_f<T>(v + gj * ld_v + h * D + d) : 0.f;
      } else {
        xs[rr][d] = in ? ld_f<T>(q + gj * ld_q + h * D + d) : 0.f;
        ys[rr][d] = in ? ld_f<T>(d_o + gj * ld_do + h * D + d) : 0.f;
      }
    }
    if (threadIdx.x < kKvChunk) {
      const int j = c0 + threadIdx.x;
      tss[threadIdx.x] = (g.ts != nullptr && j < p_end) ? g.ts[it.row0 + j] : 0;
    }
    __syncthreads();
    if (!valid) continue;
    for (int rr = 0; rr < kKvChunk; ++rr) {
      const int p = c0 + rr;
      if (p >= p_end) break;
      const int qi = (KIND == 0) ? r : p;   // query index of the pair
      const int kj = (KIND == 0) ? p : r;   // key index of the pair
      if (!visible(qi, kj, n)) continue;
      float qk = 0.f, dov = 0.f;
#pragma unroll
      for (int d = 0; d < D; ++d) {
        qk = fmaf(a[d], xs[rr][d], qk);
        if (KIND != 2) dov = fmaf(b[d], ys[rr][d], dov);
      }
      const long long t_q = (KIND == 0) ? tr : tss[rr];
      const long long t_k = (KIND == 0) ? tss[rr] : tr;
      const PairBias pb = pair_bias(g, qi, kj, n, t_q, t_k, it.row0);
      const float s = g.alpha * qk + pb.value;
      if (KIND == 2) {
        const float pa = silu_f(s);
#pragma unroll
        for (int d = 0; d < D; ++d) acc[d] = fmaf(pa, ys[rr][d], acc[d]);
      } else {
        const float ds = dov * silu_grad_f(s);
#pragma unroll
        for (int d = 0; d < D; ++d) acc[d] = fmaf(ds, xs[rr][d], acc[d]);
        if (KIND == 0) {
          if (pb.pidx >= 0) atomicAdd(&bias_grad[pb.pidx], ds);
          if (pb.tidx >= 0 && ntime > 0) atomicAdd(&bias_grad[npos + pb.tidx], ds);
          if (pb.yidx >= 0) atomicAdd(&bias_grad[npos + ntime + pb.yidx], ds);
        }
      }
    }
  }
  if (valid) {
    const float scale = (KIND == 2) ? 1.f : g.alpha;
    const int64_t ld_out_row = grow * ld_out + h * D;
#pragma unroll
    for (int d = 0; d < D; ++d) st_f<T>(out + ld_out_row + d, scale * acc[d]);
  }
  if (KIND == 0) {
    __syncthreads();
    for (int e = threadIdx.x; e < npos; e += blockDim.x)
      if (bias_grad[e] != 0.f) atomicAdd(&d_pos[e], bias_grad[e]);
    for (int e = threadIdx.x; e < ntime; e += blockDim.x)
      if (bias_grad[npos + e] != 0.f) atomicAdd(&d_time[e], bias_grad[npos + e]);
    for (int e = threadIdx.x; e < ntype; e += blockDim.x)
      if (bias_grad[npos + ntime + e] != 0.f && g.d_type != nullptr)
        atomicAdd(&g.d_type[e], bias_grad[npos + ntime + e]);
  }
}

// ---------------------------------------------------------------------------- launchers
template <typename T, int D>
static cudaError_t fwd_simt_d(const AttnGeom& g, const void* q, int64_t ld_q, const void* k,
                              int64_t ld_k, const void* v, int64_t ld_v, void* o, int64_t ld_o,
                              int grid, cudaStream_t stream) {
  attn_fwd_simt_kernel<T, D><<<grid, 128, 0, stream>>>(
      g, static_cast<const T*>(q), ld_q, static_cast<const T*>(k), ld_k,
      static_cast<const T*>(v), ld_v, static_cast<T*>(o), ld_o);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t fwd_simt_t(int D, const AttnGeom& g, const void* q, int64_t ld_q,
                              const void* k, int64_t ld_k, const void* v, int64_t ld_v, void* o,
                              int64_t ld_o, int grid, cudaStream_t stream) {
  switch (D) {
    case 16: return fwd_simt_d<T, 16>(g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, stream);
    case 32: return fwd_simt_d<T, 32>(g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, stream);
    case 64: return fwd_simt_d<T, 64>(g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, stream);
    case 128: return fwd_simt_d<T, 128>(g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_fwd_simt(int dtype, int D, const AttnGeom& g, const void* q, int64_t ld_q,
                                 const void* k, int64_t ld_k, const void* v, int64_t ld_v,
                                 void* o, int64_t ld_o, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  if (dtype == 0)
    return fwd_simt_t<__nv_bfloat16>(D, g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, stream);
  return fwd_simt_t<float>(D, g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, stream);
}

cudaError_t launch_gemm_simt(int dtype, int epi, const void* A, int64_t lda, const void* B,
                             int64_t ldb, int M, int N, int K, const float* bias, const void* R,
                             int64_t ldr, void* C, int64_t ldc, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  dim3 grid((N + 63) / 64, (M + 63) / 64);
#define HSTU_GEMM_SIMT(T, E)                                                                  \
  gemm_simt_kernel<T, E><<<grid, 256, 0, stream>>>(                                           \
      static_cast<const T*>(A), lda, static_cast<const T*>(B), ldb, M, N, K, bias,            \
      static_cast<const T*>(R), ldr, static_cast<T*>(C), ldc)
  if (dtype == 0) {
    if (epi == 0) HSTU_GEMM_SIMT(__nv_bfloat16, 0);
    else HSTU_GEMM_SIMT(__nv_bfloat16, 1);
  } else {
    if (epi == 0) HSTU_GEMM_SIMT(float, 0);
    else HSTU_GEMM_SIMT(float, 1);
  }
#undef HSTU_GEMM_SIMT
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t bwd_simt_d(const AttnGeom& g, const void* q, int64_t ld_q, const void* k,
                              int64_t ld_k, const void* v, int64_t ld_v, const void* d_o,
                              int64_t ld_do, void* dq, void* dk, void* dv, float* d_pos,
                              float* d_time, int grid, cudaStream_t stream) {
  const size_t bias_smem =
      sizeof(float) * (((g.rab_pos != nullptr) ? 2 * g.P + 1 : 0) +
                       ((g.ts != nullptr && g.rab_time != nullptr) ? g.NB : 0) +
                       ((g.rab_type != nullptr) ? g.NT * g.NT : 0));
  if (bias_smem > 200 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_bwd_simt_kernel<T, D, 0>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(bias_smem));
  if (e != cudaSuccess) return e;
  const T* tq = static_cast<const T*>(q);
  const T* tk = static_cast<const T*>(k);
  const T* tv = static_cast<const T*>(v);
  const T* tdo = static_cast<const T*>(d_o);
  attn_bwd_simt_kernel<T, D, 0><<<grid, 128, bias_smem, stream>>>(
      g, tq, ld_q, tk, ld_k, tv, ld_v, tdo, ld_do, static_cast<T*>(dq), ld_q, d_pos, d_time);
  attn_bwd_simt_kernel<T, D, 1><<<grid, 128, 0, stream>>>(
      g, tq, ld_q, tk, ld_k, tv, ld_v, tdo, ld_do, static_cast<T*>(dk), ld_k, d_pos, d_time);
  attn_bwd_simt_kernel<T, D, 2><<<grid, 128, 0, stream>>>(
      g, tq, ld_q, tk, ld_k, tv, ld_v, tdo, ld_do, static_cast<T*>(dv), ld_v, d_pos, d_time);
  return cudaGetLastError();
}

template <typename T>
static cudaError_t bwd_simt_t(int D, const AttnGeom& g, const void* q, int64_t ld_q,
                              const void* k, int64_t ld_k, const void* v, int64_t ld_v,
                              const void* d_o, int64_t ld_do, void* dq, void* dk, void* dv,
                              float* d_pos, float* d_time, int grid, cudaStream_t stream) {
  switch (D) {
    case 16: return bwd_simt_d<T, 16>(g, q, ld_q, k, ld_k, v, ld_v, d_o, ld_do, dq, dk, dv, d_pos, d_time, grid, stream);
    case 32: return bwd_simt_d<T, 32>(g, q, ld_q, k, ld_k, v, ld_v, d_o, ld_do, dq, dk, dv, d_pos, d_time, grid, stream);
    case 64: return bwd_simt_d<T, 64>(g, q, ld_q, k, ld_k, v, ld_v, d_o, ld_do, dq, dk, dv, d_pos, d_time, grid, stream);
    case 128: return bwd_simt_d<T, 128>(g, q, ld_q, k, ld_k, v, ld_v, d_o, ld_do, dq, dk, dv, d_pos, d_time, grid, stream);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_attn_bwd_simt(int dtype, int D, const AttnGeom& g, const void* q, int64_t ld_q,
                                 const void* k, int64_t ld_k, const void* v, int64_t ld_v,
                                 const void* d_o, int64_t ld_do, void* dq, void* dk, void* dv,
                                 float* d_pos, float* d_time, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  if (dtype == 0)
    return bwd_simt_t<__nv_bfloat16>(D, g, q, ld_q, k, ld_k, v, ld_v, d_o, ld_do, dq, dk, dv,
                                     d_pos, d_time, grid, stream);
  return bwd_simt_t<float>(D, g, q, ld_q, k, ld_k, v, ld_v, d_o, ld_do, dq, dk, dv, d_pos,
                           d_time, grid, stream);
}

}  // namespace hstu
