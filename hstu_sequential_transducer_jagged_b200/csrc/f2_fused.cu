// f2_fused.cu — Y = X + (Norm(AV) ⊙ U) W2 + b2 in one kernel: the gated LayerNorm is formed in
// shared memory as the tensor cores' A operand, so G never goes through HBM.
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, third formula Y = f2(Norm(AV) ⊙ U)
// and the block diagram's residual edge; "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 3.)
//
// Persistent CTAs walk 128-row blocks of tokens.  The block's AV rows [128, F] (F = H d_v <= 512)
// sit in F / 64 K-major, 128-byte-swizzled slots of [128 rows][64 features] — already the MMA's
// A-operand layout — and each slot turns into the matching slot of G in place:
//   warp 0      TMA: AV slot kb of the next block as soon as this block's MMAs have read slot kb;
//               U slots (same swizzle) through a 2-slot ring; W2 tiles [64 k][256 n] through a
//               2-stage ring, interleaved with the U slots in K order;
//   warps 2-5   one token row per thread: mean and biased variance of the row over all slots
//               (two passes over shared memory), then slot by slot as U arrives,
//               G = ((AV - mean) rstd γ + β) ⊙ U written in place as bf16, fenced for the
//               tensor core's async proxy, and published per slot;
//   warp 1      tcgen05.mma: K block kb of G against both 256-wide halves of W2 (N <= 512) into
//               two TMEM accumulators (2 x 256 columns); the slot is released after both;
//   warps 6-13  epilogue: TMEM -> + b2 + X -> bf16 Y, one row per thread, 128 of every 256
//               columns per warp; the accumulators are free again for the next block after it.
// So the next block's AV streams in while this block's MMAs run, and its statistics overlap this
// block's epilogue.
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kRows = 128;
constexpr int kTileN = 256;
constexpr int kKB = 64;
constexpr int kSlotBytes = kRows * kKB * 2;     // 16 KB: one K block of AV / G
constexpr int kBStageBytes = kKB * kTileN * 2;  // 32 KB: four [64 k][64 n] boxes of W2
constexpr int kBStages = 2;
constexpr int kUSlots = 2;
constexpr int kMaxF = 512;                      // 8 slots: 128 KB
constexpr int kMaxSlots = kMaxF / kKB;
constexpr int kMaxN = 2 * kTileN;               // two TMEM accumulators
constexpr int kThreads = 448;                   // 14 warps

struct F2Smem {
  alignas(1024) uint8_t g[kMaxSlots][kSlotBytes];
  alignas(1024) uint8_t u[kUSlots][kSlotBytes];
  alignas(1024) uint8_t b[kBStages][kBStageBytes];
  uint64_t av_full[kMaxSlots];    // TMA: slot kb holds the block's AV
  uint64_t g_ready[kMaxSlots];    // transform warps: slot kb holds G
  uint64_t slot_free[kMaxSlots];  // MMA: slot kb has been read (both halves)
  uint64_t u_full[kUSlots], u_empty[kUSlots];
  uint64_t b_full[kBStages], b_empty[kBStages];
  uint64_t acc_full, acc_empty;
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

// Lane 0 waits, the warp follows (every lane then sees what the barrier published).
__device__ __forceinline__ bool warp_wait_bar(uint64_t* bar, uint32_t parity, volatile int* abort,
                                              int* status) {
  const int lane = threadIdx.x & 31;
  return warp_all(lane == 0 ? mbar_wait(bar, parity, abort, status) : true);
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
  const int n_halves = (N + kTileN - 1) / kTileN;  // 1 or 2
  const int blocks = (M + kRows - 1) / kRows;
  const int stride = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMaxSlots; ++s) {
      mbar_init(&sm.av_full[s], 1);
      mbar_init(&sm.g_ready[s], 4);  // one elected lane per transform warp
      mbar_init(&sm.slot_free[s], 1);
    }
    for (int s = 0; s < kUSlots; ++s) {
      mbar_init(&sm.u_full[s], 1);
      mbar_init(&sm.u_empty[s], 4);
    }
    for (int s = 0; s < kBStages; ++s) {
      mbar_init(&sm.b_full[s], 1);
      mbar_init(&sm.b_empty[s], 1);
    }
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.acc_empty, 8);  // one elected lane per epilogue warp
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
      int av_slots = 0;           // AV slot loads issued
      bool ok = true;
      for (int blk = blockIdx.x; ok && blk < blocks; blk += stride, ++it) {
        for (int kb = 0; kb < nkb; ++kb) {
          // the previous block's MMAs have read slot kb
          if (it > 0 && !mbar_wait(&sm.slot_free[kb], (it - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.av_full[kb], kSlotBytes);
          tma_load_2d(sm.g[kb], &tm_av, &sm.av_full[kb], kb * kKB, blk * kRows);
          ++av_slots;
        }
        for (int kb = 0; ok && kb < nkb; ++kb) {
          const int su = gu % kUSlots;
          if (gu >= kUSlots &&
              !mbar_wait(&sm.u_empty[su], ((gu / kUSlots) - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.u_full[su], kSlotBytes);
          tma_load_2d(sm.u[su], &tm_u, &sm.u_full[su], kb * kKB, blk * kRows);
          ++gu;
          for (int h = 0; h < n_halves; ++h, ++g) {
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
                          h * kTileN + 64 * q, kb * kKB);
          }
        }
      }
      if (!ok) {  // leave no TMA write in flight into shared memory about to be released
        for (int k2 = (g > kBStages ? g - kBStages : 0); k2 < g; ++k2)
          mbar_wait(&sm.b_full[k2 % kBStages], (k2 / kBStages) & 1, nullptr, nullptr);
        for (int k2 = (gu > kUSlots ? gu - kUSlots : 0); k2 < gu; ++k2)
          mbar_wait(&sm.u_full[k2 % kUSlots], (k2 / kUSlots) & 1, nullptr, nullptr);
        // the last load of each slot (loads go to slots 0, 1, .., nkb - 1, 0, 1, ..)
        for (int s = 0; s < nkb && s < av_slots; ++s) {
          const int loads = (av_slots - 1 - s) / nkb + 1;
          mbar_wait(&sm.av_full[s], (loads - 1) & 1, nullptr, nullptr);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTileN, 0, 1);
      const uint64_t db0 = smem_desc_sw128(smem_u32(sm.b[0]), kKB * 128, 1024);
      int it = 0, g = 0;
      bool ok = true;
      for (int blk = blockIdx.x; ok && blk < blocks; blk += stride, ++it) {
        // the epilogue has read the accumulators of the previous block
        if (it > 0 && !mbar_wait(&sm.acc_empty, (it - 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kb = 0; ok && kb < nkb; ++kb) {
          if (!mbar_wait(&sm.g_ready[kb], it & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(smem_u32(sm.g[kb]), 16, 1024);
          for (int h = 0; h < n_halves; ++h, ++g) {
            const int st = g % kBStages;
            if (!mbar_wait(&sm.b_full[st], (g / kBStages) & 1, abort_flag, status)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint64_t db = db0 + static_cast<uint64_t>(st) * (kBStageBytes >> 4);
            const uint32_t d = tmem + 256u * h;
#pragma unroll
            for (int kk = 0; kk < kKB / 16; ++kk)
              mma_bf16_ss(d, da + 2 * kk, db + 128 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
            mma_commit(&sm.b_empty[st]);
          }
          if (ok) mma_commit(&sm.slot_free[kb]);  // both halves have read G slot kb
        }
        if (ok) mma_commit(&sm.acc_full);
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
      // (eight partial sums per pass: the row's 512 additions form eight short dependency
      // chains instead of one long one)
      float part[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) part[e] = 0.f;
      for (int kb = 0; ok && kb < nkb; ++kb) {
        ok = warp_wait_bar(&sm.av_full[kb], it & 1, abort_flag, status);
        if (!ok) break;
        const uint8_t* base = sm.g[kb] + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
          bf16x8_to_f(*reinterpret_cast<const uint4*>(base + ((c ^ sw) << 4)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) part[e] += f[e];
        }
      }
      if (!ok) break;
      const float mean =
          (((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]))) / F;
#pragma unroll
      for (int e = 0; e < 8; ++e) part[e] = 0.f;
      for (int kb = 0; kb < nkb; ++kb) {
        const uint8_t* base = sm.g[kb] + r * 128;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          float f[8];
          bf16x8_to_f(*reinterpret_cast<const uint4*>(base + ((c ^ sw) << 4)), f);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float dl = f[e] - mean;
            part[e] = fmaf(dl, dl, part[e]);
          }
        }
      }
      const float sq =
          ((part[0] + part[1]) + (part[2] + part[3])) + ((part[4] + part[5]) + (part[6] + part[7]));
      const float rstd = rsqrtf(sq / F + eps);
      for (int kb = 0; ok && kb < nkb; ++kb, ++gu) {
        const int su = gu % kUSlots;
        ok = warp_wait_bar(&sm.u_full[su], (gu / kUSlots) & 1, abort_flag, status);
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
        fence_async_smem();  // slot kb of G is read by the MMAs (async proxy)
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.u_empty[su]);  // this warp is done with the U slot
          mbar_arrive(&sm.g_ready[kb]);
        }
      }
    }
  } else {
    // --------------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int half = (warp - 6) >> 2;  // columns 128 half .. +127 of each 256-wide accumulator
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 128u * half;
    int it = 0;
    for (int blk = blockIdx.x; blk < blocks; blk += stride, ++it) {
      const int row = blk * kRows + quad * 32 + lane;
      const bool row_ok = row < M;
      if (!warp_all(mbar_wait(&sm.acc_full, it & 1, abort_flag, status))) break;
      tc_fence_after();
      for (int h = 0; h < n_halves; ++h) {
        const int n0 = h * kTileN + 128 * half;
        // the residual rows of this half, all loads in flight before the first use
        uint4 xr[16];
#pragma unroll
        for (int v = 0; v < 16; ++v) {
          const int c = n0 + 8 * v;
          xr[v] = (row_ok && c + 8 <= N)
                      ? *reinterpret_cast<const uint4*>(x + static_cast<int64_t>(row) * ld_x + c)
                      : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t acc[32];
          tmem_ld32(lane_addr + 256u * h + ch * 32, acc);
          tmem_wait_ld();
          const int c0 = n0 + ch * 32;
          if (row_ok && c0 < N) {
            float vals[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              float v = __uint_as_float(acc[e]);
              if (bias != nullptr && c0 + e < N) v += __ldg(bias + c0 + e);
              vals[e] = v;
            }
            __nv_bfloat16* yp = y + static_cast<int64_t>(row) * ld_y + c0;
            if (c0 + 32 <= N) {
#pragma unroll
              for (int w = 0; w < 4; ++w) {
                float fx[8];
                bf16x8_to_f(xr[4 * ch + w], fx);
                uint4 ov;
                ov.x = pack_bf16x2(vals[8 * w + 0] + fx[0], vals[8 * w + 1] + fx[1]);
                ov.y = pack_bf16x2(vals[8 * w + 2] + fx[2], vals[8 * w + 3] + fx[3]);
                ov.z = pack_bf16x2(vals[8 * w + 4] + fx[4], vals[8 * w + 5] + fx[5]);
                ov.w = pack_bf16x2(vals[8 * w + 6] + fx[6], vals[8 * w + 7] + fx[7]);
                reinterpret_cast<uint4*>(yp)[w] = ov;
              }
            } else {
              const __nv_bfloat16* xp = x + static_cast<int64_t>(row) * ld_x + c0;
              for (int e = 0; e < 32; ++e)
                if (c0 + e < N) yp[e] = __float2bfloat16_rn(vals[e] + __bfloat162float(xp[e]));
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty);
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

// Shared memory of the fused kernel.
size_t f2_fused_smem() { return sizeof(F2Smem) + 1024; }

// True when the fused kernel takes a layer: F a multiple of 64 up to 512, N a multiple of 8 up
// to 512 (two TMEM accumulators); the caller checks bf16 and 16-byte alignment.
bool f2_fused_supported(int F, int N) {
  return F % kKB == 0 && F >= kKB && F <= kMaxF && N % 8 == 0 && N >= 8 && N <= kMaxN &&
         f2_fused_smem() <= 227 * 1024;
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
