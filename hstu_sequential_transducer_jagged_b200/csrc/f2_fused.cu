// f2_fused.cu — Y = X + (Norm(AV) ⊙ U) W2 + b2 with the gated LayerNorm formed in shared memory as
// the tensor cores' A operand, so G never goes through HBM.
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, third formula Y = f2(Norm(AV) ⊙ U)
// and the block diagram's residual edge; "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 3.)
//
// The LayerNorm statistics of each row come either from the attention kernel, which leaves the
// mean and the sum of squared deviations of every 32-column slice of its output (combined here
// with the pairwise formula: mean = average of the slice means, M2 = Σ M2_s + 32 Σ (mean_s -
// mean)²), or from row_stats, one warp per row (two passes over values held in registers).
// Then the fused GEMM, a
// streaming pipeline over work units of 128 token rows x 256 output columns (units of the same
// row block sit next to each other, so the second unit's AV and U reads hit L2):
//   warp 0      TMA: per K block of 64 features, the unit's AV slot [128][64] and U slot (both
//               K-major, 128-byte swizzle, the MMA's A layout) and W2's [64 k][256 n] tile
//               through a 3-stage ring;
//   warps 2-9   G = ((AV - mean) rstd γ + β) ⊙ U in place of the AV slot (bf16), fenced for the
//               tensor core's async proxy and published per stage; two threads per row, each
//               with 32 of the slot's 64 features;
//   warp 1      tcgen05.mma of the stage's G against W2 into one of two TMEM accumulators
//               [128 x 256] fp32, so one unit's epilogue overlaps the next unit's main loop;
//   warps 10-13 epilogue: TMEM -> + b2 + X -> bf16 Y, one row per thread, in 32 x 32 chunks
//               staged in swizzled shared memory: X arrives there by TMA one chunk ahead, Y
//               leaves by TMA store (whole 64-byte rows per copy instead of warp-wide
//               accesses to 32 cache lines).
#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kRows = 128;
constexpr int kTileN = 256;
constexpr int kKB = 64;
constexpr int kSlotBytes = kRows * kKB * 2;     // 16 KB: one K block of AV / G or of U
constexpr int kBBytes = kKB * kTileN * 2;       // 32 KB: four [64 k][64 n] boxes of W2
constexpr int kStages = 3;
constexpr int kXformWarps = 8;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kXformWarps + kEpiWarps);  // 448: 128 registers a thread
constexpr int kMaxF = 1024;
constexpr int kStageTile = 32 * 32 * 2;  // 2 KB: 32 rows x 32 bf16, 64-byte swizzle

struct F2Smem {
  alignas(1024) uint8_t a[kStages][kSlotBytes];
  alignas(1024) uint8_t u[kStages][kSlotBytes];
  alignas(1024) uint8_t b[kStages][kBBytes];
  alignas(1024) uint8_t stage[kEpiWarps][2][kStageTile];
  uint64_t full[kStages];     // TMA: AV, U and W2 of the stage have landed
  uint64_t g_ready[kStages];  // transform warps: the stage's G is in place
  uint64_t empty[kStages];    // MMA: the stage has been read
  uint64_t acc_full[2], acc_empty[2];
  uint64_t xbar[kEpiWarps][2];  // residual chunk landed in stage[w][b]
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

// Mean and 1/sqrt(biased variance + eps) of each row of AV [rows, F] (F % 8 == 0, F <= 1024):
// one warp per row, 8-feature vectors, values kept in registers for the centred second pass.
__global__ void row_stats_kernel(const __nv_bfloat16* __restrict__ av, int64_t ld_av, int rows,
                                 int F, float eps, float2* __restrict__ stats) {
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const __nv_bfloat16* a = av + static_cast<int64_t>(row) * ld_av;
  float x[4][8];
  float sum = 0.f;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    const int c = (s * 32 + lane) * 8;
    const uint4 raw = c < F ? *reinterpret_cast<const uint4*>(a + c) : make_uint4(0u, 0u, 0u, 0u);
    bf16x8_to_f(raw, x[s]);
#pragma unroll
    for (int e = 0; e < 8; ++e) sum += x[s][e];
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
  const float mean = sum / F;
  float sq = 0.f;
#pragma unroll
  for (int s = 0; s < 4; ++s) {
    if ((s * 32 + lane) * 8 < F) {
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float dl = x[s][e] - mean;
        sq = fmaf(dl, dl, sq);
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
  if (lane == 0) stats[row] = make_float2(mean, rsqrtf(sq / F + eps));
}

__global__ void __launch_bounds__(kThreads, 1)
    f2_fused_kernel(const __grid_constant__ CUtensorMap tm_av,
                    const __grid_constant__ CUtensorMap tm_u,
                    const __grid_constant__ CUtensorMap tm_w2,
                    const __grid_constant__ CUtensorMap tm_x,
                    const __grid_constant__ CUtensorMap tm_y, int M, int N, int F,
                    const float2* __restrict__ stats, int nparts, float eps,
                    const float* __restrict__ gamma, const float* __restrict__ beta,
                    const float* __restrict__ bias, int* status) {
  if (*reinterpret_cast<volatile int*>(status) == kStatusTimeout) return;
  extern __shared__ uint8_t smem_raw[];
  F2Smem& sm = *reinterpret_cast<F2Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nkb = (F + kKB - 1) / kKB;
  const int nh = (N + kTileN - 1) / kTileN;
  const int units = ((M + kRows - 1) / kRows) * nh;
  const int stride = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.g_ready[s], kXformWarps);  // one elected lane per transform warp
      mbar_init(&sm.empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.acc_full[s], 1);
      mbar_init(&sm.acc_empty[s], kEpiWarps);  // one elected lane per epilogue warp
    }
    for (int w = 0; w < kEpiWarps; ++w) {
      mbar_init(&sm.xbar[w][0], 1);
      mbar_init(&sm.xbar[w][1], 1);
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
      int g = 0;  // stages issued
      bool ok = true;
      for (int un = blockIdx.x; ok && un < units; un += stride) {
        const int blk = un / nh, h = un - blk * nh;
        // W2 boxes that start past column N are not loaded: they only feed accumulator
        // columns that the epilogue never stores.
        const int nbox = min(kTileN / 64, (N - h * kTileN + 63) / 64);
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % kStages;
          if (g >= kStages &&
              !mbar_wait(&sm.empty[s], ((g / kStages) - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[s], 2 * kSlotBytes + nbox * (kKB * 128));
          tma_load_2d(sm.a[s], &tm_av, &sm.full[s], kb * kKB, blk * kRows);
          tma_load_2d(sm.u[s], &tm_u, &sm.full[s], kb * kKB, blk * kRows);
          for (int q = 0; q < nbox; ++q)
            tma_load_2d(sm.b[s] + q * (kKB * 128), &tm_w2, &sm.full[s], h * kTileN + 64 * q,
                        kb * kKB);
        }
      }
      if (!ok)  // leave no TMA write in flight into shared memory about to be released
        for (int k2 = (g > kStages ? g - kStages : 0); k2 < g; ++k2)
          mbar_wait(&sm.full[k2 % kStages], (k2 / kStages) & 1, nullptr, nullptr);
    }
    __syncwarp();
  } else if (warp == 1) {
    // --------------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kRows, kTileN, 0, 1);
      int g = 0, j = 0;
      bool ok = true;
      for (int un = blockIdx.x; ok && un < units; un += stride, ++j) {
        const int acc = j & 1;
        // the epilogue has read this accumulator's previous unit
        if (j >= 2 && !mbar_wait(&sm.acc_empty[acc], ((j >> 1) - 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + 256u * acc;
        for (int kb = 0; kb < nkb; ++kb, ++g) {
          const int s = g % kStages;
          if (!mbar_wait(&sm.g_ready[s], (g / kStages) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t da = smem_desc_sw128(smem_u32(sm.a[s]), 16, 1024);
          const uint64_t db = smem_desc_sw128(smem_u32(sm.b[s]), kKB * 128, 1024);
#pragma unroll
          for (int kk = 0; kk < kKB / 16; ++kk)
            mma_bf16_ss(d, da + 2 * kk, db + 128 * kk, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(&sm.empty[s]);
        }
        if (ok) mma_commit(&sm.acc_full[acc]);
      }
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else if (warp < 2 + kXformWarps) {
    // --------------------------------------------------------------------- Norm(AV) ⊙ U
    const int t = warp - 2;
    const int r = (t & 3) * 32 + lane;  // row of the unit
    const int c_lo = (t >> 2) * 4;      // 16-byte chunks c_lo .. c_lo + 3 of each slot
    const int sw = r & 7;               // 128-byte swizzle: chunk c sits at c ^ (r & 7)
    const bool vec_gb = (gamma == nullptr || (reinterpret_cast<uintptr_t>(gamma) & 15) == 0) &&
                        (beta == nullptr || (reinterpret_cast<uintptr_t>(beta) & 15) == 0) &&
                        F % 8 == 0;
    int g = 0;
    bool ok = true;
    for (int un = blockIdx.x; ok && un < units; un += stride) {
      const int row = (un / nh) * kRows + r;
      float2 st = make_float2(0.f, 0.f);  // (mean, rstd); rows past M: zero
      if (row < M) {
        if (nparts == 0) {
          st = stats[row];
        } else {
          // the slices' (mean, M2) pairs, 32 values each, merged in order (Chan et al.)
          const float2* ps = stats + static_cast<int64_t>(row) * nparts;
          float mean = 0.f, m2 = 0.f, n = 0.f;
          for (int i = 0; i < nparts; ++i) {
            const float2 p = ps[i];
            const float n2 = n + 32.f;
            const float dl = p.x - mean;
            mean = fmaf(dl, 32.f / n2, mean);
            m2 += p.y + dl * dl * (n * 32.f / n2);
            n = n2;
          }
          st = make_float2(mean, rsqrtf(m2 / F + eps));
        }
      }
      const float2 rs2 = make_float2(st.y, st.y);
      const float2 sh2 = make_float2(-st.x * st.y, -st.x * st.y);  // (v - mean) rstd = v rstd + sh
      for (int kb = 0; kb < nkb; ++kb, ++g) {
        const int s = g % kStages;
        ok = warp_wait_bar(&sm.full[s], (g / kStages) & 1, abort_flag, status);
        if (!ok) break;
        uint8_t* base = sm.a[s] + r * 128;
        const uint8_t* ubase = sm.u[s] + r * 128;
        uint4 araw[4], uraw[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int off = ((c_lo + c) ^ sw) << 4;
          araw[c] = *reinterpret_cast<const uint4*>(base + off);
          uraw[c] = *reinterpret_cast<const uint4*>(ubase + off);
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = kb * kKB + (c_lo + c) * 8;
          float gv[8], bv[8];
          if (vec_gb && col < F) {
            const float4 g0 = gamma ? __ldg(reinterpret_cast<const float4*>(gamma + col)) : make_float4(1.f, 1.f, 1.f, 1.f);
            const float4 g1 = gamma ? __ldg(reinterpret_cast<const float4*>(gamma + col + 4)) : make_float4(1.f, 1.f, 1.f, 1.f);
            const float4 b0 = beta ? __ldg(reinterpret_cast<const float4*>(beta + col)) : make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 b1 = beta ? __ldg(reinterpret_cast<const float4*>(beta + col + 4)) : make_float4(0.f, 0.f, 0.f, 0.f);
            gv[0] = g0.x; gv[1] = g0.y; gv[2] = g0.z; gv[3] = g0.w;
            gv[4] = g1.x; gv[5] = g1.y; gv[6] = g1.z; gv[7] = g1.w;
            bv[0] = b0.x; bv[1] = b0.y; bv[2] = b0.z; bv[3] = b0.w;
            bv[4] = b1.x; bv[5] = b1.y; bv[6] = b1.z; bv[7] = b1.w;
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {  // features past F: U is zero there (TMA fill)
              const bool in = col + e < F;
              gv[e] = (in && gamma) ? __ldg(gamma + col + e) : 1.f;
              bv[e] = (in && beta) ? __ldg(beta + col + e) : 0.f;
            }
          }
          const __nv_bfloat162* ah = reinterpret_cast<const __nv_bfloat162*>(&araw[c]);
          const __nv_bfloat162* uh = reinterpret_cast<const __nv_bfloat162*>(&uraw[c]);
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 av2 = __bfloat1622float2(ah[e]);
            const float2 u2 = __bfloat1622float2(uh[e]);
            const float2 nv = fma2(fma2(av2, rs2, sh2), make_float2(gv[2 * e], gv[2 * e + 1]),
                                   make_float2(bv[2 * e], bv[2 * e + 1]));
            w[e] = pack_bf16x2(nv.x * u2.x, nv.y * u2.y);
          }
          *reinterpret_cast<uint4*>(base + (((c_lo + c) ^ sw) << 4)) =
              make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_async_smem();  // the stage's G is read by the MMAs (async proxy)
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.g_ready[s]);
      }
    }
  } else {
    // --------------------------------------------------------------------- epilogue
    const int ew = warp - 2 - kXformWarps;
    const int quad = warp & 3;  // TMEM lanes 32 quad .. 32 quad + 31 (the warp's sub-partition)
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const bool bias_vec = bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
    uint8_t* stg0 = sm.stage[ew][0];
    uint8_t* stg1 = sm.stage[ew][1];
    // one wait follows each residual load of a buffer: bit b of xph is the parity of buffer b's
    // next completion, bit b of pend marks a load not yet waited for
    uint32_t xph = 0, pend = 0;
    int j = 0;
    bool ok = true;
    for (int un = blockIdx.x; ok && un < units; un += stride, ++j) {
      const int acc = j & 1;
      const int blk = un / nh, h = un - blk * nh;
      const int r0 = blk * kRows + quad * 32;
      const int n0 = h * kTileN;
      // the first residual chunk (buffer 0's last store has read it)
      if (lane == 0) {
        bulk_wait_read<1>();
        mbar_arrive_expect_tx(&sm.xbar[ew][0], kStageTile);
        tma_load_2d(stg0, &tm_x, &sm.xbar[ew][0], n0, r0);
      }
      pend |= 1u;
      if (!warp_all(mbar_wait(&sm.acc_full[acc], (j >> 1) & 1, abort_flag, status))) {
        ok = false;
        break;
      }
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < kTileN / 32; ++ch) {
        const int c0 = n0 + ch * 32;
        if (c0 >= N) break;  // warp-uniform
        const int xb = ch & 1;
        uint8_t* stg = xb ? stg1 : stg0;
        uint32_t accv[32];
        tmem_ld32(lane_addr + 256u * acc + ch * 32, accv);
        tmem_wait_ld();
        ok = warp_all(lane == 0 ? mbar_wait(&sm.xbar[ew][xb], (xph >> xb) & 1u, abort_flag, status)
                                : true);
        if (!ok) break;
        xph ^= 1u << xb;
        pend &= ~(1u << xb);
        float bv[32];
        if (bias == nullptr) {
#pragma unroll
          for (int e = 0; e < 32; ++e) bv[e] = 0.f;
        } else if (bias_vec && c0 + 32 <= N) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) {
            const float4 b4 = __ldg(reinterpret_cast<const float4*>(bias + c0 + e));
            bv[e] = b4.x;
            bv[e + 1] = b4.y;
            bv[e + 2] = b4.z;
            bv[e + 3] = b4.w;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) bv[e] = c0 + e < N ? __ldg(bias + c0 + e) : 0.f;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint4* slot = reinterpret_cast<uint4*>(stg + stage64_offset(lane, q));
          const uint4 xr = *slot;
          const __nv_bfloat162* x2 = reinterpret_cast<const __nv_bfloat162*>(&xr);
          uint32_t o[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 f = __bfloat1622float2(x2[e]);
            const int k0 = 8 * q + 2 * e;
            o[e] = pack_bf16x2(__uint_as_float(accv[k0]) + bv[k0] + f.x,
                               __uint_as_float(accv[k0 + 1]) + bv[k0 + 1] + f.y);
          }
          *slot = make_uint4(o[0], o[1], o[2], o[3]);
        }
        fence_proxy_async_smem();  // the staging tile is read by the TMA store
        __syncwarp();
        if (lane == 0) {
          if (r0 < M) {  // rows past M and columns past N are clipped
            tma_store_2d(&tm_y, stg, c0, r0);
            bulk_commit();
          }
          if (ch + 1 < kTileN / 32 && c0 + 32 < N) {
            // the previous chunk's store has read the other buffer: the next residual chunk
            bulk_wait_read<1>();
            mbar_arrive_expect_tx(&sm.xbar[ew][xb ^ 1], kStageTile);
            tma_load_2d(xb ? stg0 : stg1, &tm_x, &sm.xbar[ew][xb ^ 1], c0 + 32, r0);
          }
        }
        if (ch + 1 < kTileN / 32 && c0 + 32 < N) pend |= 1u << (xb ^ 1);
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[acc]);
    }
    if (lane == 0) {
      // after a timeout: no residual load still writing into the staging tiles
      for (int b2 = 0; b2 < 2; ++b2)
        if (pend & (1u << b2)) mbar_wait(&sm.xbar[ew][b2], (xph >> b2) & 1u, nullptr, nullptr);
      bulk_wait_all();  // the staging tiles stay valid until the stores are done
    }
    __syncwarp();
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

// True when the fused kernel takes a layer: F and N multiples of 8 (16-byte rows for TMA and the
// vector loads) and F <= 1024 (the statistics kernel keeps a row in one warp's registers); the
// caller checks bf16 and 16-byte alignment.
bool f2_fused_supported(int F, int N) {
  return F % 8 == 0 && F >= 8 && F <= kMaxF && N % 8 == 0 && N >= 8 &&
         f2_fused_smem() <= 227 * 1024;
}

// nparts = 0: `stats` is scratch for M float2 (mean, rstd) rows, written by a first launch;
// nparts > 0 (= F / 32): `stats` holds the attention kernel's per-slice (mean, M2) pairs.
// tm_x / tm_y: X and Y [M, N], 32 x 32 boxes, 64-byte swizzle.
cudaError_t launch_f2_fused(const CUtensorMap& tm_av, const CUtensorMap& tm_u,
                            const CUtensorMap& tm_w2, const CUtensorMap& tm_x,
                            const CUtensorMap& tm_y, const __nv_bfloat16* av, int64_t ld_av,
                            int M, int N, int F, const float* gamma, const float* beta, float eps,
                            const float* bias, float2* stats, int nparts, int* status,
                            int num_sms, cudaStream_t stream) {
  if (M <= 0 || N <= 0) return cudaSuccess;
  if (!f2_fused_supported(F, N) || (nparts != 0 && nparts * 32 != F)) return cudaErrorInvalidValue;
  const int st_threads = 256;
  if (nparts == 0)
  row_stats_kernel<<<static_cast<unsigned>((static_cast<int64_t>(M) * 32 + st_threads - 1) / st_threads),
                     st_threads, 0, stream>>>(
      av, ld_av, M, F, eps, stats);
  const size_t smem = f2_fused_smem();
  cudaError_t e = cudaFuncSetAttribute(f2_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int units = ((M + kRows - 1) / kRows) * ((N + kTileN - 1) / kTileN);
  const int grid = units < num_sms ? units : num_sms;
  f2_fused_kernel<<<grid, kThreads, smem, stream>>>(tm_av, tm_u, tm_w2, tm_x, tm_y, M, N, F,
                                                   stats, nparts, eps, gamma, beta, bias, status);
  return cudaGetLastError();
}

}  // namespace hstu
