// gemm_tc.cu — the two single linear layers of the HSTU layer on the 5th-generation tensor cores.
//
//   f1:  Z = SiLU(X W1 + b1)            (φ1(f1(X)), then Split into U, V, Q, K by column block)
//   f2:  Y = X + G W2 + b2              (G = Norm(AV) ⊙ U; the residual edge of the block diagram)
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1: f1, f2 single linear layers,
//  φ1 = SiLU; the residual edge from the input to the output.)
//
// C[M, N] = epilogue(A[M, K] · B[K, N]) with A row-major (K-major operand) and B row-major
// (the weight as stored, an MN-major operand), bf16 in, fp32 accumulate in TMEM, bf16 out.
// Persistent: one CTA per SM walks the 128 x 256 output tiles with a fixed stride.  Tiles are
// 128 x 256 x 64 per K block (four N = 256 MMAs), through a 4-stage TMA ring that runs on
// across tiles; the accumulator is double-buffered in TMEM (2 x 256 columns), so the epilogue
// of one tile overlaps the main loop of the next.  Warp 0 TMA producer, warp 1 TMEM allocation
// + single-thread tcgen05.mma issue, warps 2..9 epilogue: warp w reads TMEM lanes 32 (w % 4)
// .. +31 (one output row per thread) and columns 128 ((w - 2) / 4) .. +127 of the tile.
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kBM = 128;
constexpr int kBN = 256;
constexpr int kBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmThreads = 320;  // 10 warps
constexpr int kABytes = kBM * kBK * 2;   // 16 KB: [128 rows][64 k], SW128, K-major
constexpr int kBBytes = kBK * kBN * 2;   // 32 KB: four [64 k][64 n] SW128 boxes, MN-major

struct GemmSmem {
  alignas(1024) uint8_t a[kGemmStages][kABytes];
  alignas(1024) uint8_t b[kGemmStages][kBBytes];
  uint64_t full[kGemmStages];
  uint64_t empty[kGemmStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

// SiLU(x) = x σ(x) = h (1 + tanh h) with h = x / 2: one MUFU operation per element.
__device__ __forceinline__ float silu_fast(float x) {
  const float h = 0.5f * x;
  return fmaf(h, tanh_fast(h), h);
}

}  // namespace

// EPI 0: C = SiLU(acc + bias);  EPI 1: C = acc + bias + R (residual, bf16 [M, N], ld_r).
template <int EPI>
__global__ void __launch_bounds__(kGemmThreads, 1)
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
  const int kblocks = (K + kBK - 1) / kBK;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int tiles = ((M + kBM - 1) / kBM) * n_tiles;
  const int stride = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], 8);  // one elected lane per epilogue warp
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

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_a);
      tma_prefetch_desc(&tm_b);
      int g = 0;  // K blocks issued so far (the ring runs on across tiles)
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += stride) {
        const int m0 = (t / n_tiles) * kBM;
        const int n0 = (t % n_tiles) * kBN;
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const int st = g % kGemmStages;
          if (g >= kGemmStages &&
              !mbar_wait(&sm.empty[st], ((g / kGemmStages) - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[st], kABytes + kBBytes);
          tma_load_2d(sm.a[st], &tm_a, &sm.full[st], kb * kBK, m0);
#pragma unroll
          for (int q = 0; q < kBN / 64; ++q)
            tma_load_2d(sm.b[st] + q * (kBK * 128), &tm_b, &sm.full[st], n0 + 64 * q, kb * kBK);
        }
      }
      if (!ok) {  // leave no TMA write in flight into shared memory about to be released
        for (int k2 = (g > kGemmStages ? g - kGemmStages : 0); k2 < g; ++k2)
          mbar_wait(&sm.full[k2 % kGemmStages], (k2 / kGemmStages) & 1, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, 0, 1);
      const uint64_t da0 = smem_desc_sw128(smem_u32(sm.a[0]), 16, 1024);
      const uint64_t db0 = smem_desc_sw128(smem_u32(sm.b[0]), kBK * 128, 1024);
      int g = 0, j = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += stride, ++j) {
        const int ab = j & 1;
        // the epilogue has read this accumulator buffer's previous tile
        if (j >= 2 && !mbar_wait(&sm.acc_empty[ab], ((j - 2) >> 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + 256u * ab;
        for (int kb = 0; kb < kblocks; ++kb, ++g) {
          const int st = g % kGemmStages;
          if (!mbar_wait(&sm.full[st], (g / kGemmStages) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = da0 + static_cast<uint64_t>(st) * (kABytes >> 4);
          const uint64_t db = db0 + static_cast<uint64_t>(st) * (kBBytes >> 4);
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk)
            mma_bf16_ss(d, da + 2 * kk, db + 128 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.empty[st]);
        }
        if (ok) mma_commit(&sm.acc_full[ab]);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int half = (warp - 2) >> 2;  // columns 128 * half .. +127 of the tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 128u * half;
    int j = 0;
    for (int t = blockIdx.x; t < tiles; t += stride, ++j) {
      const int ab = j & 1;
      const int m0 = (t / n_tiles) * kBM;
      const int n0 = (t % n_tiles) * kBN + 128 * half;
      const int row = m0 + quad * 32 + lane;
      if (!warp_all(mbar_wait(&sm.acc_full[ab], (j >> 1) & 1, abort_flag, status))) break;
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < 128 / 32; ++ch) {
        uint32_t acc[32];
        tmem_ld32(lane_addr + 256u * ab + ch * 32, acc);
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
            for (int e = 0; e < 32; ++e) vals[e] = silu_fast(vals[e]);
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
      // this warp's part of the accumulator buffer is read: the MMA warp may reuse it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_gemm_bf16_tc(int epi, const CUtensorMap& ta, const CUtensorMap& tb, int M,
                                int N, int K, const float* bias, const __nv_bfloat16* resid,
                                int64_t ld_r, __nv_bfloat16* C, int64_t ldc, int* status,
                                cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  const size_t smem = sizeof(GemmSmem) + 1024;
  const int tiles = ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN);
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = tiles < sms ? tiles : sms;
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
