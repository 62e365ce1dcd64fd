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
// The bf16 epilogues write each 32 x 32 chunk into a swizzled shared-memory staging tile
// (two per warp) and store it with one TMA store, and the residual arrives the same way, one
// chunk ahead: a row per thread but whole 64-byte rows per copy, instead of warp-wide
// accesses that touch 32 cache lines each.
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
constexpr int kEpiWarps = 8;
constexpr int kStageTile = 32 * 32 * 2;  // 2 KB: 32 rows x 32 bf16, 64-byte swizzle

struct GemmSmem {
  alignas(1024) uint8_t a[kGemmStages][kABytes];
  alignas(1024) uint8_t b[kGemmStages][kBBytes];
  alignas(1024) uint8_t stage[kEpiWarps][2][kStageTile];
  uint64_t rbar[kEpiWarps][2];  // residual chunk landed in stage[w][b]
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

// Operand layouts (template parameters):
//   A_MN = 0: A is stored [M, K] row-major (K-major operand): one box {64 k, 128 m} per stage.
//   A_MN = 1: A is stored [K, M] row-major (MN-major operand, e.g. Gᵀ of a [T, F] activation):
//             two boxes {64 m, 64 k} per stage, 8 KB apart.
//   B_MN = 1: B is stored [K, N] row-major (MN-major): four boxes {64 n, 64 k}, 8 KB apart.
//   B_MN = 0: B is stored [N, K] row-major (K-major, e.g. Wᵀ of a stored weight): one box
//             {64 k, 256 n}.
// Epilogues:
//   EPI 0: C = SiLU(acc + bias)                       (bf16)
//   EPI 1: C = acc + bias + R                         (bf16, residual R [M, N] with ld_r)
//   EPI 2: C = acc + bias                             (bf16)
//   EPI 3: C = SiLU(acc + bias) and C2 = acc + bias   (bf16 C; fp32 C2 with ld_c2: the
//          pre-activation the backward's SiLU' reads)
//   EPI 4: Cf += acc                                  (fp32, atomic: split-K partial sums)
// With k_splits > 1 each output tile is computed by k_splits work units over consecutive K
// ranges (EPI 4 only).
template <int EPI, int A_MN, int B_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tm_a,
                        const __grid_constant__ CUtensorMap tm_b,
                        const __grid_constant__ CUtensorMap tm_c,
                        const __grid_constant__ CUtensorMap tm_r, int M, int N, int K,
                        int k_splits, const float* __restrict__ bias,
                        const __nv_bfloat16* __restrict__ resid, int64_t ld_r,
                        __nv_bfloat16* __restrict__ C, int64_t ldc,
                        float* __restrict__ C2, int64_t ld_c2, float* __restrict__ Cf,
                        int* status) {
  if (*reinterpret_cast<volatile int*>(status) == kStatusTimeout) return;
  extern __shared__ uint8_t smem_raw[];
  GemmSmem& sm = *reinterpret_cast<GemmSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int kblocks = (K + kBK - 1) / kBK;
  const int kb_per = (kblocks + k_splits - 1) / k_splits;
  const int n_tiles = (N + kBN - 1) / kBN;
  const int mn_tiles = ((M + kBM - 1) / kBM) * n_tiles;
  const int tiles = mn_tiles * k_splits;
  const int stride = static_cast<int>(gridDim.x);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], kEpiWarps);  // one elected lane per epilogue warp
    }
    for (int w = 0; w < kEpiWarps; ++w) {
      mbar_init(&sm.rbar[w][0], 1);
      mbar_init(&sm.rbar[w][1], 1);
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
        const int mn = t % mn_tiles, ks = t / mn_tiles;
        const int m0 = (mn / n_tiles) * kBM;
        const int n0 = (mn % n_tiles) * kBN;
        const int kb1 = min(kblocks, (ks + 1) * kb_per);
        for (int kb = ks * kb_per; kb < kb1; ++kb, ++g) {
          const int st = g % kGemmStages;
          if (g >= kGemmStages &&
              !mbar_wait(&sm.empty[st], ((g / kGemmStages) - 1) & 1, abort_flag, status)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&sm.full[st], kABytes + kBBytes);
          if (A_MN) {
#pragma unroll
            for (int q = 0; q < kBM / 64; ++q)
              tma_load_2d(sm.a[st] + q * (kBK * 128), &tm_a, &sm.full[st], m0 + 64 * q, kb * kBK);
          } else {
            tma_load_2d(sm.a[st], &tm_a, &sm.full[st], kb * kBK, m0);
          }
          if (B_MN) {
#pragma unroll
            for (int q = 0; q < kBN / 64; ++q)
              tma_load_2d(sm.b[st] + q * (kBK * 128), &tm_b, &sm.full[st], n0 + 64 * q, kb * kBK);
          } else {
            tma_load_2d(sm.b[st], &tm_b, &sm.full[st], kb * kBK, n0);
          }
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
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, kBN, A_MN, B_MN);
      // K-major: the next 16 k are 32 bytes further in the swizzled row; MN-major: 16 rows of
      // 128 bytes further, with the 64-wide M (N) chunks kBK x 128 bytes apart
      const uint64_t da0 = A_MN ? smem_desc_sw128(smem_u32(sm.a[0]), kBK * 128, 1024)
                                : smem_desc_sw128(smem_u32(sm.a[0]), 16, 1024);
      const uint64_t db0 = B_MN ? smem_desc_sw128(smem_u32(sm.b[0]), kBK * 128, 1024)
                                : smem_desc_sw128(smem_u32(sm.b[0]), 16, 1024);
      constexpr uint64_t a_step = A_MN ? 128 : 2;
      constexpr uint64_t b_step = B_MN ? 128 : 2;
      int g = 0, j = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += stride, ++j) {
        const int ks = t / mn_tiles;
        const int kb0 = ks * kb_per, kb1 = min(kblocks, (ks + 1) * kb_per);
        const int ab = j & 1;
        // the epilogue has read this accumulator buffer's previous tile
        if (j >= 2 && !mbar_wait(&sm.acc_empty[ab], ((j - 2) >> 1) & 1, abort_flag, status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + 256u * ab;
        for (int kb = kb0; kb < kb1; ++kb, ++g) {
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
            mma_bf16_ss(d, da + a_step * kk, db + b_step * kk, idesc,
                        (kb > kb0 || kk > 0) ? 1u : 0u);
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
    const int ew = warp - 2;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16) + 128u * half;
    const bool bias_vec = bias != nullptr && (reinterpret_cast<uintptr_t>(bias) & 15) == 0;
    uint8_t* stg0 = sm.stage[ew][0];
    uint8_t* stg1 = sm.stage[ew][1];
    // residual loads: one wait follows each load of a buffer; bit b of rph is the parity of
    // buffer b's next completion, bit b of pend marks a load not yet waited for
    uint32_t rph = 0, pend = 0;
    int j = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < tiles; t += stride, ++j) {
      const int ab = j & 1;
      const int mn = t % mn_tiles, ks = t / mn_tiles;
      const int m0 = (mn / n_tiles) * kBM;
      const int n0 = (mn % n_tiles) * kBN + 128 * half;
      const int r0 = m0 + quad * 32;  // first row of this warp's 32
      const int row = r0 + lane;
      if constexpr (EPI == 1) {
        // the first residual chunk: buffer 0's last store (chunk 2 of the previous tile) has
        // read it
        if (n0 < N) {
          if (lane == 0) {
            bulk_wait_read<1>();
            mbar_arrive_expect_tx(&sm.rbar[ew][0], kStageTile);
            tma_load_2d(stg0, &tm_r, &sm.rbar[ew][0], n0, r0);
          }
          pend |= 1u;
        }
      }
      if (!warp_all(mbar_wait(&sm.acc_full[ab], (j >> 1) & 1, abort_flag, status))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // a K range past the end (k_splits not dividing the K blocks) contributed nothing
      const bool empty_range = ks * kb_per >= kblocks;
#pragma unroll 1
      for (int ch = 0; ch < 128 / 32; ++ch) {
        uint32_t acc[32];
        tmem_ld32(lane_addr + 256u * ab + ch * 32, acc);
        tmem_wait_ld();
        const int c0 = n0 + ch * 32;
        if constexpr (EPI == 4) {
          if (row < M && c0 < N && !empty_range) {
            float* cp = Cf + static_cast<int64_t>(row) * ldc + c0;
            if (c0 + 32 <= N) {
#pragma unroll
              for (int e = 0; e < 32; e += 4)
                atomicAdd(reinterpret_cast<float4*>(cp + e),
                          make_float4(__uint_as_float(acc[e]), __uint_as_float(acc[e + 1]),
                                      __uint_as_float(acc[e + 2]), __uint_as_float(acc[e + 3])));
            } else {
              for (int e = 0; e < 32; ++e)
                if (c0 + e < N) atomicAdd(cp + e, __uint_as_float(acc[e]));
            }
          }
        } else {
          if (c0 >= N) continue;  // warp-uniform: nothing of this chunk is stored
          uint8_t* stg = (ch & 1) ? stg1 : stg0;
          float vals[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) vals[e] = __uint_as_float(acc[e]);
          if (bias != nullptr) {
            if (bias_vec && c0 + 32 <= N) {
#pragma unroll
              for (int e = 0; e < 32; e += 4) {
                const float4 bv = __ldg(reinterpret_cast<const float4*>(bias + c0 + e));
                vals[e] += bv.x;
                vals[e + 1] += bv.y;
                vals[e + 2] += bv.z;
                vals[e + 3] += bv.w;
              }
            } else {
#pragma unroll
              for (int e = 0; e < 32; ++e)
                if (c0 + e < N) vals[e] += __ldg(bias + c0 + e);
            }
          }
          if (EPI == 3 && row < M) {  // the fp32 pre-activation, before the SiLU overwrites vals
            float* pp = C2 + static_cast<int64_t>(row) * ld_c2 + c0;
            if (c0 + 32 <= N) {
#pragma unroll
              for (int w = 0; w < 8; ++w)
                reinterpret_cast<float4*>(pp)[w] = make_float4(vals[4 * w], vals[4 * w + 1],
                                                               vals[4 * w + 2], vals[4 * w + 3]);
            } else {
              for (int e = 0; e < 32; ++e)
                if (c0 + e < N) pp[e] = vals[e];
            }
          }
          if constexpr (EPI == 1) {
            // this chunk's residual rows (TMA, zero past the bounds), then the next chunk's
            const int rb = ch & 1;
            ok = warp_all(lane == 0 ? mbar_wait(&sm.rbar[ew][rb], (rph >> rb) & 1u, abort_flag,
                                                status)
                                    : true);
            if (!ok) break;
            rph ^= 1u << rb;
            pend &= ~(1u << rb);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const uint4 rv = *reinterpret_cast<const uint4*>(stg + stage64_offset(lane, q));
              const __nv_bfloat162* r2 = reinterpret_cast<const __nv_bfloat162*>(&rv);
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 f = __bfloat1622float2(r2[e]);
                vals[8 * q + 2 * e] += f.x;
                vals[8 * q + 2 * e + 1] += f.y;
              }
            }
          } else {
            // the store two chunks back has read this buffer
            if (lane == 0) bulk_wait_read<1>();
            __syncwarp();
            if (EPI == 0 || EPI == 3) {
#pragma unroll
              for (int e = 0; e < 32; ++e) vals[e] = silu_fast(vals[e]);
            }
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 ov;
            ov.x = pack_bf16x2(vals[8 * q + 0], vals[8 * q + 1]);
            ov.y = pack_bf16x2(vals[8 * q + 2], vals[8 * q + 3]);
            ov.z = pack_bf16x2(vals[8 * q + 4], vals[8 * q + 5]);
            ov.w = pack_bf16x2(vals[8 * q + 6], vals[8 * q + 7]);
            *reinterpret_cast<uint4*>(stg + stage64_offset(lane, q)) = ov;
          }
          fence_proxy_async_smem();  // the staging tile is read by the TMA store
          __syncwarp();
          if (lane == 0) {
            if (r0 < M) {  // rows past M and columns past N are clipped
              tma_store_2d(&tm_c, stg, c0, r0);
              bulk_commit();
            }
            if constexpr (EPI == 1) {
              if (ch + 1 < 128 / 32 && c0 + 32 < N) {
                // the previous chunk's store has read the other buffer: the next residual
                bulk_wait_read<1>();
                uint8_t* nxt = (ch & 1) ? stg0 : stg1;
                mbar_arrive_expect_tx(&sm.rbar[ew][(ch + 1) & 1], kStageTile);
                tma_load_2d(nxt, &tm_r, &sm.rbar[ew][(ch + 1) & 1], c0 + 32, r0);
              }
            }
          }
          if (EPI == 1 && ch + 1 < 128 / 32 && c0 + 32 < N) pend |= 1u << ((ch + 1) & 1);
        }
      }
      if (!ok) break;
      // this warp's part of the accumulator buffer is read: the MMA warp may reuse it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.acc_empty[ab]);
    }
    if (lane == 0) {
      // after a timeout: no residual load still writing into the staging tiles
      for (int b2 = 0; b2 < 2; ++b2)
        if (pend & (1u << b2)) mbar_wait(&sm.rbar[ew][b2], (rph >> b2) & 1u, nullptr, nullptr);
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

namespace {
template <int EPI, int A_MN, int B_MN>
cudaError_t launch_gemm_t(const GemmArgs& a, int grid, size_t smem, cudaStream_t stream) {
  auto kern = gemm_bf16_tc_kernel<EPI, A_MN, B_MN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kGemmThreads, smem, stream>>>(*a.ta, *a.tb, *a.tc, *a.tr, a.M, a.N, a.K,
                                             a.k_splits, a.bias,
                                             a.resid, a.ld_r, a.C, a.ldc, a.C2, a.ld_c2, a.Cf,
                                             a.status);
  return cudaGetLastError();
}
}  // namespace

// Tiles of one launch for the given shape, before split-K.
int gemm_tc_mn_tiles(int M, int N) { return ((M + kBM - 1) / kBM) * ((N + kBN - 1) / kBN); }

cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream) {
  if (a.M <= 0 || a.N <= 0) return cudaSuccess;
  if (a.k_splits < 1 || (a.k_splits > 1 && a.epi != 4)) return cudaErrorInvalidValue;
  const size_t smem = sizeof(GemmSmem) + 1024;
  const int tiles = gemm_tc_mn_tiles(a.M, a.N) * a.k_splits;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = tiles < sms ? tiles : sms;
  const int key = a.epi * 4 + a.a_mn * 2 + a.b_mn;
  switch (key) {
    case 0 * 4 + 0 * 2 + 1: return launch_gemm_t<0, 0, 1>(a, grid, smem, stream);  // f1 + SiLU
    case 1 * 4 + 0 * 2 + 1: return launch_gemm_t<1, 0, 1>(a, grid, smem, stream);  // f2 + residual
    case 3 * 4 + 0 * 2 + 1: return launch_gemm_t<3, 0, 1>(a, grid, smem, stream);  // f1, pre kept
    case 2 * 4 + 0 * 2 + 0: return launch_gemm_t<2, 0, 0>(a, grid, smem, stream);  // dY W2^T
    case 1 * 4 + 0 * 2 + 0: return launch_gemm_t<1, 0, 0>(a, grid, smem, stream);  // dY + dZ W1^T
    case 4 * 4 + 1 * 2 + 1: return launch_gemm_t<4, 1, 1>(a, grid, smem, stream);  // X^T dZ
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace hstu
