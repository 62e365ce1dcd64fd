// gemm_tc.cu — the two single linear layers of the HSTU layer on the 5th-generation tensor cores.
//
//   f1:  Z = SiLU(X W1 + b1)            (φ1(f1(X)), then Split into U, V, Q, K by column block)
//   f2:  Y = X + G W2 + b2              (G = Norm(AV) ⊙ U; the residual edge of the block diagram)
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1: f1, f2 single linear layers,
//  φ1 = SiLU; the residual edge from the input to the output.)
//
// C[M, N] = epilogue(A[M, K] · B[K, N]) with A row-major (K-major operand) and B row-major
// (the weight as stored, an MN-major operand), bf16 in, fp32 accumulate in TMEM, bf16 out.
// Tile 128 x 128 x 64, 3-stage TMA ring, one CTA per output tile, two CTAs per SM so that one
// CTA's epilogue overlaps the other's main loop.  Warp roles as in the attention kernel:
// warp 0 TMA producer, warp 1 TMEM allocation + single-thread tcgen05.mma issue,
// warps 2..5 epilogue (one thread per output row, tcgen05.ld of 32 columns at a time).
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 128;
constexpr int kBK = 64;
constexpr int kGemmStages = 3;
constexpr int kGemmThreads = 192;

struct GemmSmem {
  alignas(1024) uint8_t a[kGemmStages][kBM * kBK * 2];  // [128 rows][64 k] SW128, K-major
  alignas(1024) uint8_t b[kGemmStages][kBK * kBN * 2];  // two [64 k][64 n] SW128 boxes
  uint64_t full[kGemmStages];
  uint64_t empty[kGemmStages];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ float silu_accurate(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

}  // namespace

// EPI 0: C = SiLU(acc + bias);  EPI 1: C = acc + bias + R (residual, bf16 [M, N], ld_r).
template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 2)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b, int M, int N, int K,
                        const float* __restrict__ bias, const __nv_bfloat16* __restrict__ resid,
                        int64_t ld_r, __nv_bfloat16* __restrict__ C, int64_t ldc,
                        int* status) {
  if (*reinterpret_cast<volatile int*>(status) == kStatusTimeout) return;
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kBN;
  const int m0 = blockIdx.y * kBM;
  const int kblocks = (K + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      int issued = 0;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int st = kb % kGemmStages;
        if (kb >= kGemmStages &&
            !mbar_wait(&sm.empty[st], ((kb / kGemmStages) - 1) & 1, abort_flag, status))
          break;
        mbar_arrive_expect_tx(&sm.full[st], (kBM * kBK + kBK * kBN) * 2);
        tma_load_2d(sm.a[st], &tm_a, &sm.full[st], kb * kBK, m0);
        tma_load_2d(sm.b[st], &tm_b, &sm.full[st], n0, kb * kBK);
        tma_load_2d(sm.b[st] + kBK * 128, &tm_b, &sm.full[st], n0 + 64, kb * kBK);
        issued = kb + 1;
      }
      if (*abort_flag) {
        for (int kb = (issued > kGemmStages ? issued - kGemmStages : 0); kb < issued; ++kb)
          mbar_wait(&sm.full[kb % kGemmStages], (kb / kGemmStages) & 1, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 1);
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int st = kb % kGemmStages;
        if (!mbar_wait(&sm.full[st], (kb / kGemmStages) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(sm.a[st]);
        const uint32_t b_base = smem_u32(sm.b[st]);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk) {
          mma_bf16_ss(tmem, smem_desc_sw128(a_base + kk * 32, 16, 1024),
                      smem_desc_sw128(b_base + kk * 2048, kBK * 128, 1024), idesc,
                      (kb > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.empty[st]);
      }
      mma_commit(&sm.acc_full);
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else {
    const int quad = warp & 3;
    const int row = m0 + quad * 32 + lane;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    if (warp_all(mbar_wait(&sm.acc_full, 0, abort_flag, status))) {
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < kBN / 32; ++ch) {
        uint32_t acc[32];
        tmem_ld32(lane_addr + ch * 32, acc);
        tmem_wait_ld();
        const int c0 = n0 + ch * 32;
        if (row < M && c0 < N) {
          float vals[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = c0 + e;
            float x = __uint_as_float(acc[e]);
            if (bias != nullptr && c < N) x += __ldg(bias + c);
            vals[e] = x;
          }
          if (EPI == 1) {
            const __nv_bfloat16* rp = resid + static_cast<int64_t>(row) * ld_r + c0;
            if (c0 + 32 <= N) {
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                uint4 rv = *reinterpret_cast<const uint4*>(rp + 8 * w);
                const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rv);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  float2 f = __bfloat1622float2(r2[e]);
                  vals[8 * w + 2 * e] += f.x;
                  vals[8 * w + 2 * e + 1] += f.y;
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c0 + e < N) vals[e] += __bfloat162float(rp[e]);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) vals[e] = silu_accurate(vals[e]);
          }
          __nv_bfloat16* cp = C + static_cast<int64_t>(row) * ldc + c0;
          if (c0 + 32 <= N) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              uint4 ov;
              ov.x = pack_bf16x2(vals[8 * w + 0], vals[8 * w + 1]);
              ov.y = pack_bf16x2(vals[8 * w + 2], vals[8 * w + 3]);
              ov.z = pack_bf16x2(vals[8 * w + 4], vals[8 * w + 5]);
              ov.w = pack_bf16x2(vals[8 * w + 6], vals[8 * w + 7]);
              reinterpret_cast<uint4*>(cp)[w] = ov;
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              if (c0 + e < N) cp[e] = __float2bfloat16_rn(vals[e]);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
  }
}

cudaError_t launch_gemm_bf16_tc(int epi, const CUtensorMap& ta, const CUtensorMap& tb, int M,
                                int N, int K, const float* bias, const __nv_bfloat16* resid,
                                int64_t ld_r, __nv_bfloat16* C, int64_t ldc, int* status,
                                cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const size_t smem = sizeof(GemmSmem) + 1024;
  dim3 grid((N + kBN - 1) / kBN, (M + kBM - 1) / kBM);
  cudaError_t e;
  if (epi == 0) {
    e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    gemm_bf16_tc_kernel<0><<<grid, kGemmThreads, smem, stream>>>(ta, tb, M, N, K, bias, resid,
                                                                  ld_r, C, ldc, status);
  } else {
    e = cudaFuncSetAttribute(gemm_bf16_tc_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)smem);
    if (e != cudaSuccess) return e;
    gemm_bf16_tc_kernel<1><<<grid, kGemmThreads, smem, stream>>>(ta, tb, M, N, K, bias, resid,
                                                                  ld_r, C, ldc, status);
  }
  return cudaGetLastError();
}

}  // namespace hstu
