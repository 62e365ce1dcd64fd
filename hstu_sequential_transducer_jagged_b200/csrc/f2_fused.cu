// f2_fused.cu — Y = X + (Norm(AV) ⊙ U) W2 + b2 in one kernel: the gated LayerNorm is formed in
// shared memory as the tensor cores' A operand, so G never goes through HBM.
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, third formula Y = f2(Norm(AV) ⊙ U)
// and the block diagram's residual edge; "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 3.)
//
// Persistent CTAs walk 128-row blocks of tokens.  Per block:
//   warp 0      TMA: the block's AV rows [128, F] (F = H d_v <= 512) into shared memory, as
//               F / 64 K-major 128-byte-swizzled slots of [128 rows][64 features] — already the
//               A operand's layout; the matching U slots (same swizzle) through a 2-slot ring;
//               then W2 tiles [64 k][256 n] through a 2-stage ring;
//   warps 2-5   one token row per thread: mean and biased variance of the row from shared memory
//               (two passes), then, slot by slot as U arrives, G = ((AV - mean) rstd γ + β) ⊙ U
//               written in place as bf16, fenced for the tensor core's async proxy;
//   warp 1      tcgen05.mma: for each 256-wide output tile, F / 64 K blocks of four 128x256x16
//               MMAs into one of two TMEM accumulators (2 x 256 columns);
//   warps 6-13  epilogue: TMEM -> + b2 + X -> bf16 Y, one row per thread, 128 columns per warp.
// The next block's AV load waits for this block's last MMA (one G buffer); the accumulators are
// double-buffered, so the epilogue of one tile overlaps the MMAs of the next.
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kRows = 128;
constexpr int kTileN = 256;
constexpr int kKB = 64;
constexpr int kSlotBytes = kRows * kKB * 2;   // 16 KB: one K block of G
constexpr int kBStageBytes = kKB * kTileN * 2; // 32 KB: four [64 k][64 n] boxes of W2
constexpr int kBStages = 2;
constexpr int kUSlots = 2;
constexpr int kMaxF = 512;                     // 8 slots: 128 KB
constexpr int kThreads = 448;                  // 14 warps

struct F2Smem {
  alignas(1024) uint8_t g[kMaxF / kKB][kSlotBytes];
  alignas(1024) uint8_t u[kUSlots][kSlotBytes];
  alignas(1024) uint8_t b[kBStages][kBStageBytes];
  uint64_t g_loaded, g_ready, g_free;
  uint64_t u_full[kUSlots], u_empty[kUSlots];
  uint64_t b_full[kBStages], b_empty[kBStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void bf16x8_to_f(const uint4& raw, float (&f)[8]) {
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 v = __bfloat1622float2(h[e]);
    f[2 * e] = v.x;
    f[2 * e + 1] = v.y;
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    f2_fused_kernel(const __grid_constant__ CUtensorMap tm_av,
                    const __grid_constant__ CUtensorMap tm_u,
                    const __grid_constant__ CUtensorMap tm_w2, int M, int N, int F,
                    const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                    const float* __restrict__ bias, const __nv_bfloat16* __restrict__ x,
                    int64_t ld_x, __nv_bfloat16* __restrict__ y, int64_t ld_y, int* status) {
  if (*reinterpret_cast<volatile int*>(status) == kStatusTimeout) return;
  extern __shared__ uint8_t smem_raw[];
  F2Smem& sm = *reinterpret_cast<F2Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = F / kKB;
  const int n_tiles = (N + kTileN - 1) / kTileN;
  const int blocks = (M + kRows - 1) / kRows;
  const int stride = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    mbar_init(&sm.g_loaded, 1);
    mbar_init(&sm.g_ready, 4);  // one elected lane per transform warp
    mbar_init(&sm.g_free, 1);
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&sm.b_full[s], 1);
      mbar_init(&sm.b_empty[s], 1);
    }
    for (int s = 0; s < kUSlots; ++s) {
      mbar_init(&sm.u_full[s], 1);
      mbar_init(&sm.u_empty[s], 4);  // one elected lane per transform warp
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm.acc_full[a], 1);
      mbar_init(&sm.acc_empty[a], 8);
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
    // --------------------------------------------------------------------- TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tm_av);
      tma_prefetch_desc(&tm_u);
      tma_prefetch_desc(&tm_w2);
      int it = 0, g = 0, gu = 0;  // blocks, W2 stages and U slots issued
      int av_issued = 0;          // blocks whose AV slots were requested
      bool ok = true;
      for (int blk = blockIdx.x; ok && blk < blocks; blk += stride, ++it) {
        // the previous block's MMAs have read G
        if (it > 0 && !mbar_wait(&sm.g_free, (it - 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm.g_loaded, nkb * kSlotBytes);
        for (int kb = 0; kb < nkb; ++kb)
          tma_load_2d(sm.g[kb], &tm_av, &sm.g_loaded, kb * kKB, blk * kRows);
        ++av_issued;
        for (int kb = 0; kb < nkb; ++kb, ++gu) {
          const int su = gu % kUSlots;
          if (gu >= kUSlots &&
              !mbar_wait(&sm.u_empty[su], ((gu / kUSlots) - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.u_full[su], kSlotBytes);
          tma_load_2d(sm.u[su], &tm_u, &sm.u_full[su], kb * kKB, blk * kRows);
        }
        if (!ok) break;
        for (int nt = 0; ok && nt < n_tiles; ++nt) {
          for (int kb = 0; kb < nkb; ++kb, ++g) {
            const int st = g % kBStages;
            if (g >= kBStages &&
                !mbar_wait(&sm.b_empty[st], ((g / kBStages) - 1) & 1, abort_flag, status)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&sm.b_full[st], kBStageBytes);
#pragma unroll
            for (int q = 0; q < kTileN / 64; ++q)
              tma_load_2d(sm.b[st] + q * (kKB * 128), &tm_w2, &sm.b_full[st],
                          nt * kTileN + 64 * q, kb * kKB);
          }
        }
      }
      if (!ok) {  // leave no TMA write in flight into shared memory about to be released
        for (int k2 = (g > kBStages ? g - kBStages : 0); k2 < g; ++k2)
          mbar_wait(&sm.b_full[k2 % kBStages], (k2 / kBStages) & 1, nullptr, nullptr);
        for (int k2 = (gu > kUSlots ? gu - kUSlots : 0); k2 < gu; ++k2)
          mbar_wait(&sm.u_full[k2 % kUSlots], (k2 / kUSlots) & 1, nullptr, nullptr);
        if (av_issued > 0) mbar_wait(&sm.g_loaded, (av_issued - 1) & 1, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTileN, 0, 1);
      const uint64_t db0 = smem_desc_sw128(smem_u32(sm.b[0]), kKB * 128, 1024);
      int it = 0, g = 0, j = 0;
      bool ok = true;
      for (int blk = blockIdx.x; ok && blk < blocks; blk += stride, ++it) {
        if (!mbar_wait(&sm.g_ready, it & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int nt = 0; ok && nt < n_tiles; ++nt, ++j) {
          const int ab = j & 1;
          if (j >= 2 && !mbar_wait(&sm.acc_empty[ab], ((j - 2) >> 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d = tmem + 256u * ab;
          for (int kb = 0; kb < nkb; ++kb, ++g) {
            const int st = g % kBStages;
            if (!mbar_wait(&sm.b_full[st], (g / kBStages) & 1, abort_flag, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t da = smem_desc_sw128(smem_u32(sm.g[kb]), 16, 1024);
            const uint64_t db = db0 + static_cast<uint64_t>(st) * (kBStageBytes >> 4);
#pragma unroll
            for (int kk = 0; kk < kKB / 16; ++kk)
              mma_bf16_ss(d, da + 2 * kk, db + 128 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&sm.b_empty[st]);
          }
          if (ok) mma_commit(&sm.acc_full[ab]);
        }
        if (ok) mma_commit(&sm.g_free);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp < 6) {
    // --------------------------------------------------------------------- Norm(AV) ⊙ U
    const int r = (warp - 2) * 32 + lane;  // row of the block
    const int sw = r & 7;                   // 128-byte swizzle: chunk c sits at c ^ (r & 7)
    int it = 0, gu = 0;
    bool ok = true;
    for (int blk = blockIdx.x; ok && blk < blocks; blk += stride, ++it) {
      ok = warp_all(lane == 0 ? mbar_wait(&sm.g_loaded, it & 1, abort_flag, status) : true);
      if (!ok) break;
      // (every lane observes the TMA writes: the waiting lane acquired them, the vote orders
      // the warp)
      float sum = 0.f;
      for (int kb = 0; kb < nkb; ++kb) {
        const uint8_t* base = sm.g[kb] + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
          bf16x8_to_f(*reinterpret_cast<const uint4*>(base + ((c ^ sw) << 4)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) sum += f[e];
        }
      }
      const float mean = sum / F;
      float sq = 0.f;
      for (int kb = 0; kb < nkb; ++kb) {
        const uint8_t* base = sm.g[kb] + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
          bf16x8_to_f(*reinterpret_cast<const uint4*>(base + ((c ^ sw) << 4)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float dl = f[e] - mean;
            sq += dl * dl;
          }
        }
      }
      const float rstd = rsqrtf(sq / F + eps);
      for (int kb = 0; kb < nkb && ok; ++kb, ++gu) {
        const int su = gu % kUSlots;
        ok = warp_all(lane == 0 ? mbar_wait(&sm.u_full[su], (gu / kUSlots) & 1, abort_flag,
                                            status)
                                : true);
        if (!ok) break;
        uint8_t* base = sm.g[kb] + r * 128;
        const uint8_t* ubase = sm.u[su] + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint4* slot = reinterpret_cast<uint4*>(base + ((c ^ sw) << 4));
          const int col = kb * kKB + c * 8;
          float f[8], fu[8];
          bf16x8_to_f(*slot, f);
          // U past the last token is zero (TMA fill), so G is zero there too
          bf16x8_to_f(*reinterpret_cast<const uint4*>(ubase + ((c ^ sw) << 4)), fu);
          float o[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            float nv = (f[e] - mean) * rstd;
            if (gamma != nullptr) nv *= gamma[col + e];
            if (beta != nullptr) nv += beta[col + e];
            o[e] = nv * fu[e];
          }
          uint4 w;
          w.x = pack_bf16x2(o[0], o[1]);
          w.y = pack_bf16x2(o[2], o[3]);
          w.z = pack_bf16x2(o[4], o[5]);
          w.w = pack_bf16x2(o[6], o[7]);
          *slot = w;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.u_empty[su]);  // this warp is done with the U slot
      }
      if (!ok) break;
      fence_async_smem();  // G is read by the MMAs (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.g_ready);
    }
  } else {
    // --------------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int half = (warp - 6) >> 2;  // columns 128 half .. +127 of the 256-wide tile
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 128u * half;
    int j = 0;
    for (int blk = blockIdx.x; blk < blocks; blk += stride) {
      const int row = blk * kRows + quad * 32 + lane;
      bool ok = true;
      for (int nt = 0; nt < n_tiles; ++nt, ++j) {
        const int ab = j & 1;
        if (!warp_all(mbar_wait(&sm.acc_full[ab], (j >> 1) & 1, abort_flag, status))) {
          ok = false;
          break;
        }
        tc_fence_after();
        const int n0 = nt * kTileN + 128 * half;
#pragma unroll 1
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t acc[32];
          tmem_ld32(lane_addr + 256u * ab + ch * 32, acc);
          tmem_wait_ld();
          const int c0 = n0 + ch * 32;
          if (row < M && c0 < N) {
            float vals[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float v = __uint_as_float(acc[e]);
              if (bias != nullptr && c0 + e < N) v += __ldg(bias + c0 + e);
              vals[e] = v;
            }
            const __nv_bfloat16* xp = x + static_cast<int64_t>(row) * ld_x + c0;
            __nv_bfloat16* yp = y + static_cast<int64_t>(row) * ld_y + c0;
            if (c0 + 32 <= N) {
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                float fx[8];
                bf16x8_to_f(*reinterpret_cast<const uint4*>(xp + 8 * w), fx);
                uint4 ov;
                ov.x = pack_bf16x2(vals[8 * w + 0] + fx[0], vals[8 * w + 1] + fx[1]);
                ov.y = pack_bf16x2(vals[8 * w + 2] + fx[2], vals[8 * w + 3] + fx[3]);
                ov.z = pack_bf16x2(vals[8 * w + 4] + fx[4], vals[8 * w + 5] + fx[5]);
                ov.w = pack_bf16x2(vals[8 * w + 6] + fx[6], vals[8 * w + 7] + fx[7]);
                reinterpret_cast<uint4*>(yp)[w] = ov;
              }
            } else {
              for (int e = 0; e < 32; ++e)
                if (c0 + e < N) yp[e] = __float2bfloat16_rn(vals[e] + __bfloat162float(xp[e]));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
      }
      if (!ok) break;
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

// Shared memory of the fused kernel (F features per token).
size_t f2_fused_smem() { return sizeof(F2Smem) + 1024; }

// True when the fused kernel takes a layer: bf16, F a multiple of 64 up to 512, N a multiple of
// 8 (the caller also checks 16-byte alignment of the operands).
bool f2_fused_supported(int F, int N) {
  return F % kKB == 0 && F >= kKB && F <= kMaxF && N % 8 == 0 && f2_fused_smem() <= 227 * 1024;
}

cudaError_t launch_f2_fused(const CUtensorMap& tm_av, const CUtensorMap& tm_u,
                            const CUtensorMap& tm_w2, int M, int N, int F, const float* gamma,
                            const float* beta, float eps, const float* bias,
                            const __nv_bfloat16* x, int64_t ld_x, __nv_bfloat16* y, int64_t ld_y,
                            int* status, int num_sms, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (!f2_fused_supported(F, N)) return cudaErrorInvalidValue;
  const size_t smem = f2_fused_smem();
  cudaError_t e = cudaFuncSetAttribute(f2_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int blocks = (M + kRows - 1) / kRows;
  const int grid = blocks < num_sms ? blocks : num_sms;
  f2_fused_kernel<<<grid, kThreads, smem, stream>>>(tm_av, tm_u, tm_w2, M, N, F, gamma, beta,
                                                   eps, bias, x, ld_x, y, ld_y, status);
  return cudaGetLastError();
}

}  // namespace hstu
