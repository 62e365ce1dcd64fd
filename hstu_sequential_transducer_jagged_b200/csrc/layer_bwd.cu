// layer_bwd.cu — the HBM-bound steps of the HSTU layer's backward pass (the chain rule through
// Y = X + f2(Norm(A(X)V(X)) ⊙ U(X)) with U,V,Q,K = Split(SiLU(f1(X))), "万亿参数推荐大模型：HSTU
// 架构如何超越传统 Self-Attention" §2.1; the whole user sequence trained in one causal pass,
// "HSTU：Scaling Law 的首次探索" §7.1.3):
//   * the gate and LayerNorm backward, one warp per token: from AV, U and dG it forms
//     dU = dG ⊙ Norm(AV) and dAV = Norm'(dG ⊙ U) (plus the affine's dgamma / dbeta),
//   * dZ = dA ⊙ SiLU'(Z) over the f1 pre-activation Z,
//   * column sums for the bias gradients.
// The matrix products of the backward run on the tensor-core GEMM (gemm_tc.cu) and the
// attention's own backward (attn_bwd_tc.cu).
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kVec = 8;            // bf16 per 16-byte vector

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&f)[8]) {
  const uint4 raw = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __bfloat1622float2(h[e]);
    f[2 * e] = v.x;
    f[2 * e + 1] = v.y;
  }
}

__device__ __forceinline__ void store8(__nv_bfloat16* p, const float (&f)[8]) {
  uint4 o;
  o.x = pack_bf16x2(f[0], f[1]);
  o.y = pack_bf16x2(f[2], f[3]);
  o.z = pack_bf16x2(f[4], f[5]);
  o.w = pack_bf16x2(f[6], f[7]);
  *reinterpret_cast<uint4*>(p) = o;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Loads / stores PER consecutive bf16 (PER a multiple of 4) as 8-byte vectors.
template <int PER>
__device__ __forceinline__ void load_row(const __nv_bfloat16* p, float (&f)[PER]) {
#pragma unroll
  for (int v = 0; v < PER / 4; ++v) {
    const uint2 raw = reinterpret_cast<const uint2*>(p)[v];
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
    const float2 a = __bfloat1622float2(h[0]), b = __bfloat1622float2(h[1]);
    f[4 * v] = a.x;
    f[4 * v + 1] = a.y;
    f[4 * v + 2] = b.x;
    f[4 * v + 3] = b.y;
  }
}
template <int PER>
__device__ __forceinline__ void store_row(__nv_bfloat16* p, const float (&f)[PER]) {
#pragma unroll
  for (int v = 0; v < PER / 4; ++v) {
    uint2 o;
    o.x = pack_bf16x2(f[4 * v], f[4 * v + 1]);
    o.y = pack_bf16x2(f[4 * v + 2], f[4 * v + 3]);
    reinterpret_cast<uint2*>(p)[v] = o;
  }
}

// One warp per token row (grid-stride), F = 32 PER features (H*d_v), lane l owning the PER
// consecutive features from l PER.  With n = (a - mean) rstd, nt = n γ + β, G = nt ⊙ U:
//   dU = dG ⊙ nt;  d_out = dG ⊙ U;  dn = d_out ⊙ γ;
//   dAV = rstd (dn - mean(dn) - n mean(dn ⊙ n));  dγ += d_out ⊙ n;  dβ += d_out.
// dγ / dβ are summed per warp in registers and added once per warp (fp32 atomics).
template <int PER>
__global__ void ln_gate_bwd_kernel(const __nv_bfloat16* __restrict__ av, int64_t ld_av,
                                   const __nv_bfloat16* __restrict__ u, int64_t ld_u,
                                   const __nv_bfloat16* __restrict__ dg, int64_t ld_dg,
                                   const float* __restrict__ gamma, const float* __restrict__ beta,
                                   float eps, __nv_bfloat16* __restrict__ d_av, int64_t ld_dav,
                                   __nv_bfloat16* __restrict__ d_u, int64_t ld_du,
                                   const float* __restrict__ z_u, int64_t ld_z,
                                   float* __restrict__ d_gamma, float* __restrict__ d_beta,
                                   int rows) {
  constexpr int F = 32 * PER;
  const int lane = threadIdx.x & 31;
  const int c0 = lane * PER;
  const int warps = (gridDim.x * blockDim.x) >> 5;
  const bool affine_grads = d_gamma != nullptr || d_beta != nullptr;
  float acc_g[PER], acc_b[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc_g[e] = acc_b[e] = 0.f;
  for (int r = (blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows; r += warps) {
    float x[PER];
    load_row<PER>(av + static_cast<int64_t>(r) * ld_av + c0, x);
    float sum = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) sum += x[e];
    const float mean = warp_sum(sum) / F;
    float sq = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      x[e] -= mean;
      sq += x[e] * x[e];
    }
    const float rstd = rsqrtf(warp_sum(sq) / F + eps);
    float fg[PER], fu[PER], du[PER];
    load_row<PER>(dg + static_cast<int64_t>(r) * ld_dg + c0, fg);
    load_row<PER>(u + static_cast<int64_t>(r) * ld_u + c0, fu);
    float s1 = 0.f, s2 = 0.f;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const float n = x[e] * rstd;
      const float g = gamma != nullptr ? gamma[c0 + e] : 1.f;
      const float nt = beta != nullptr ? fmaf(n, g, beta[c0 + e]) : n * g;
      du[e] = fg[e] * nt;
      const float dout = fg[e] * fu[e];
      if (affine_grads) {
        acc_g[e] += dout * n;
        acc_b[e] += dout;
      }
      x[e] = n;
      fg[e] = dout * g;  // dn
      s1 += fg[e];
      s2 += fg[e] * n;
    }
    if (z_u != nullptr) {  // dpre of the U block: dU ⊙ SiLU'(Z_U), rounded once
      const float* zr = z_u + static_cast<int64_t>(r) * ld_z + c0;
#pragma unroll
      for (int e = 0; e < PER; e += 4) {
        const float4 z4 = *reinterpret_cast<const float4*>(zr + e);
        du[e] *= silu_grad_z(z4.x);
        du[e + 1] *= silu_grad_z(z4.y);
        du[e + 2] *= silu_grad_z(z4.z);
        du[e + 3] *= silu_grad_z(z4.w);
      }
    }
    store_row<PER>(d_u + static_cast<int64_t>(r) * ld_du + c0, du);
    const float m1 = warp_sum(s1) / F, m2 = warp_sum(s2) / F;
#pragma unroll
    for (int e = 0; e < PER; ++e) fu[e] = rstd * (fg[e] - m1 - x[e] * m2);
    store_row<PER>(d_av + static_cast<int64_t>(r) * ld_dav + c0, fu);
  }
  if (affine_grads) {
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (d_gamma != nullptr) atomicAdd(d_gamma + c0 + e, acc_g[e]);
      if (d_beta != nullptr) atomicAdd(d_beta + c0 + e, acc_b[e]);
    }
  }
}

// dz = da ⊙ SiLU'(z), SiLU'(z) = σ(z) (1 + z (1 - σ(z))), σ(z) = (1 + tanh(z/2)) / 2; z fp32,
// da / dz bf16, rows x cols (cols a multiple of 8, 16-byte aligned rows); dz may alias da.
__global__ void silu_grad_mul_kernel(const float* __restrict__ z, int64_t ld_z,
                                     const __nv_bfloat16* da, int64_t ld_da, __nv_bfloat16* dz,
                                     int64_t ld_dz, int rows, int cols) {
  const int per_row = cols / kVec;
  const int64_t total = static_cast<int64_t>(rows) * per_row;
  for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = idx / per_row;
    const int c = static_cast<int>(idx % per_row) * kVec;
    float fa[8], o[8];
    load8(da + r * ld_da + c, fa);
    const float4 z0 = *reinterpret_cast<const float4*>(z + r * ld_z + c);
    const float4 z1 = *reinterpret_cast<const float4*>(z + r * ld_z + c + 4);
    const float fz[8] = {z0.x, z0.y, z0.z, z0.w, z1.x, z1.y, z1.z, z1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = fa[e] * silu_grad_z(fz[e]);
    store8(dz + r * ld_dz + c, o);
  }
}

// out[c] += Σ_r m[r][c] over rows [row0, row1) of a block's slice (fp32 atomics; out zeroed by
// the caller).  One thread per column.
__global__ void colsum_kernel(const __nv_bfloat16* __restrict__ m, int64_t ld, int rows, int cols,
                              int rows_per_block, float* __restrict__ out) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= cols) return;
  const int r0 = blockIdx.y * rows_per_block;
  const int r1 = min(rows, r0 + rows_per_block);
  float s = 0.f;
  for (int r = r0; r < r1; ++r) s += __bfloat162float(m[static_cast<int64_t>(r) * ld + c]);
  if (r1 > r0) atomicAdd(out + c, s);
}

}  // namespace

cudaError_t launch_ln_gate_bwd(const __nv_bfloat16* av, int64_t ld_av, const __nv_bfloat16* u,
                               int64_t ld_u, const __nv_bfloat16* dg, int64_t ld_dg,
                               const float* gamma, const float* beta, float eps,
                               __nv_bfloat16* d_av, int64_t ld_dav, __nv_bfloat16* d_u,
                               int64_t ld_du, const float* z_u, int64_t ld_z, float* d_gamma,
                               float* d_beta, int rows, int F, int num_sms,
                               cudaStream_t stream) {
  if (rows <= 0) return cudaSuccess;
  const int threads = 256;
  int blocks = (rows * 32 + threads - 1) / threads;
  // with affine gradients every warp flushes its column sums once: cap the warps
  if ((d_gamma != nullptr || d_beta != nullptr) && blocks > num_sms * 8) blocks = num_sms * 8;
#define HSTU_LN_BWD(PER)                                                                    \
  ln_gate_bwd_kernel<PER><<<blocks, threads, 0, stream>>>(av, ld_av, u, ld_u, dg, ld_dg, gamma, \
                                                          beta, eps, d_av, ld_dav, d_u, ld_du, \
                                                          z_u, ld_z, d_gamma, d_beta, rows)
  switch (F) {
    case 128: HSTU_LN_BWD(4); break;
    case 256: HSTU_LN_BWD(8); break;
    case 512: HSTU_LN_BWD(16); break;
    case 1024: HSTU_LN_BWD(32); break;
    default: return cudaErrorInvalidValue;
  }
#undef HSTU_LN_BWD
  return cudaGetLastError();
}

cudaError_t launch_silu_grad_mul(const float* z, int64_t ld_z, const __nv_bfloat16* da,
                                 int64_t ld_da, __nv_bfloat16* dz, int64_t ld_dz, int rows,
                                 int cols, int num_sms, cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  if (cols % kVec != 0) return cudaErrorInvalidValue;
  const int64_t total = static_cast<int64_t>(rows) * (cols / kVec);
  int64_t blocks = (total + 255) / 256;
  if (blocks > static_cast<int64_t>(num_sms) * 16) blocks = static_cast<int64_t>(num_sms) * 16;
  silu_grad_mul_kernel<<<static_cast<int>(blocks), 256, 0, stream>>>(z, ld_z, da, ld_da, dz,
                                                                     ld_dz, rows, cols);
  return cudaGetLastError();
}

cudaError_t launch_colsum(const __nv_bfloat16* m, int64_t ld, int rows, int cols, float* out,
                          cudaStream_t stream) {
  if (rows <= 0 || cols <= 0) return cudaSuccess;
  cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * cols, stream);
  if (e != cudaSuccess) return e;
  const int rpb = 512;
  dim3 grid((cols + 255) / 256, (rows + rpb - 1) / rpb);
  colsum_kernel<<<grid, 256, 0, stream>>>(m, ld, rows, cols, rpb, out);
  return cudaGetLastError();
}

}  // namespace hstu
