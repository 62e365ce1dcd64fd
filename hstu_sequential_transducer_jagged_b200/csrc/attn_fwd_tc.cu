// attn_fwd_tc.cu — jagged HSTU pointwise attention forward on the 5th-generation tensor cores.
//
// Computes, per head and per 128-row query tile of a jagged sequence,
//   O_i = Σ_{j visible from i} SiLU(alpha <q_i, k_j> + rab_pos[..] + rab_time[..]) v_j
// ("万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention" §2.1, second formula; the SiLU replaces
// the softmax, "HSTU：Scaling Law 的首次探索" §7.1.4 innovation 1; no normalisation, so no running
// max/sum as in softmax attention).
//
// One CTA = one (query tile, head) work item, taken longest-first from the work list.  Warp roles:
//   warp 0      TMA producer: the Q tile once, then K/V tiles into a 2-stage ring; its lanes
//               also stage the KV tile's timestamps (with their min/max) in shared memory.
//   warp 1      allocates 256 TMEM columns; lane 0 issues tcgen05.mma:
//               S = Q Kᵀ (SS, M=128 N=128, into TMEM cols [0,128)),
//               O += P V (TS: P read from TMEM cols [128,192) as bf16, V from shared memory,
//               O in TMEM cols [192,192+D)).
//   warps 2..5  epilogue, one thread per query row (TMEM lane): tcgen05.ld of S, relative bias,
//               mask, SiLU with one MUFU op (tanh), bf16 pack, tcgen05.st of P; at the end O is
//               read from TMEM and stored as bf16.
// Whole tiles above the causal diagonal, and candidate-by-other-candidate tiles under the
// M-FALCON mask ("HSTU：Scaling Law 的首次探索" §7.1.5), are never visited.
//
// The bias is evaluated per row in three grades: a row segment whose 128 keys are all visible
// and fall in a single position bucket (distance beyond the clamp) and a single log2 time bucket
// (checked from the tile's min/max timestamp, monotonicity of the bucket rule makes that exact
// for any timestamp order) adds one constant; a fully visible segment otherwise gathers the
// bias per element from shared-memory tables; boundary segments also apply the mask.
#include <climits>

#include "common.cuh"
#include "ptx.cuh"

namespace hstu {

namespace {

constexpr int kStages = 2;
constexpr int kThreads = 192;
constexpr int kColS = 0;
constexpr int kColP = 128;
constexpr int kColO = 192;
constexpr int kPosSmemMax = 4097;  // position tables up to P = 2048 live in shared memory
constexpr int kTimeSmem = 64;      // buckets above 62 are unreachable for int64 differences

template <int D>
struct FwdSmem {
  static constexpr int kTileBytes = kTileRows * D * 2;  // one 128 x D bf16 tile
  alignas(1024) uint8_t q[kTileBytes];
  alignas(1024) uint8_t k[kStages][kTileBytes];
  alignas(1024) uint8_t v[kStages][kTileBytes];
  long long ts[kStages][kTileRows];
  long long tmin[kStages];
  long long tmax[kStages];
  float rab_time[kTimeSmem];
  uint64_t q_full;
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t s_full;
  uint64_t p_full;
  uint64_t o_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
  float rab_pos[1];  // variable length tail: 2P+1 entries when the table lives in smem
};


// Epilogue for one 32-column chunk of S (this thread's row).  MODE 0: constant bias, no mask;
// MODE 1: per-element bias, no mask; MODE 2: per-element bias and mask.
template <int D, int MODE>
__device__ __forceinline__ void silu_chunk(const uint32_t (&s)[32], uint32_t (&pk)[16],
                                           float half_alpha, float half_bias, int c_base,
                                           int i, int pi, int n, int P, const float* pos_tab,
                                           const float* time_tab, bool use_time,
                                           const long long* ts_tile, long long ti, int NB,
                                           bool row_valid, const int32_t* types_seq,
                                           const float* type_row, int L) {
#pragma unroll
  for (int e = 0; e < 32; e += 2) {
    float pv[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const float acc = __uint_as_float(s[e + u]);
      float h;
      if (MODE == 0) {
        h = fmaf(half_alpha, acc, half_bias);
      } else {
        const int c = c_base + e + u;
        const int j = c;  // key index local to the sequence (c_base is already the local column)
        float bias = 0.f;
        if (pos_tab != nullptr) {
          const int pj = j < n ? j : n;
          bias += pos_tab[pos_index_direct(pi, pj, P)];
        }
        if (use_time) bias += time_tab[time_bucket64(ti - ts_tile[c - (c_base & ~127)], NB)];
        // token-type term: type_row = rab_type + type_i * NT (keys past the sequence are masked)
        if (type_row != nullptr && j < L) bias += type_row[__ldg(types_seq + j)];
        h = fmaf(half_alpha, acc, 0.5f * bias);
      }
      float p = fmaf(h, tanh_fast(h), h);
      if (MODE == 2) {
        const int j = c_base + e + u;
        const bool vis = row_valid && (j <= i) && (j < n || j == i);
        p = vis ? p : 0.f;
      }
      pv[u] = p;
    }
    pk[e >> 1] = pack_bf16x2(pv[0], pv[1]);
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 2 : 1)
    attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q,
                       const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, AttnGeom g,
                       __nv_bfloat16* __restrict__ out, int64_t ld_o) {
  static_assert(D == 64 || D == 128, "head width");
  constexpr int kAtoms = D / 64;  // 128-byte swizzle atoms across the head width
  constexpr int kTileBytes = FwdSmem<D>::kTileBytes;
  constexpr int kColsNeeded = kColO + D;
  constexpr int kAlloc = kColsNeeded <= 256 ? 256 : 512;

  const int item_idx = blockIdx.x / g.H;
  const int head = blockIdx.x % g.H;
  if (item_idx >= *g.item_count) return;
  // a CTA that timed out earlier in this launch stream: skip the work instead of waiting again
  if (*reinterpret_cast<volatile int*>(g.status) == kStatusTimeout) return;
  const WorkItem it = g.items[item_idx];

  extern __shared__ uint8_t smem_raw[];
  FwdSmem<D>& sm = *reinterpret_cast<FwdSmem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int L = it.len;
  const int n = hist_len(L, g.mask, g.num_candidates);
  const KvRange kr = kv_range(it.qtile, L, n);
  const int nkv = kr.count();
  const bool use_time = (g.ts != nullptr) && (g.rab_time != nullptr);
  const bool pos_in_smem = (g.rab_pos != nullptr) && (2 * g.P + 1 <= kPosSmemMax);
  const float* pos_tab = g.rab_pos == nullptr ? nullptr : (pos_in_smem ? sm.rab_pos : g.rab_pos);

  // ---- setup: tables to shared memory, barriers, TMEM allocation
  if (pos_in_smem)
    for (int e = threadIdx.x; e < 2 * g.P + 1; e += kThreads) sm.rab_pos[e] = g.rab_pos[e];
  if (use_time)
    for (int e = threadIdx.x; e < kTimeSmem; e += kThreads)
      sm.rab_time[e] = g.rab_time[e < g.NB ? e : g.NB - 1];
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    mbar_init(&sm.s_full, 1);
    mbar_init(&sm.p_full, 4 * 32);
    mbar_init(&sm.o_full, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, kAlloc);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;
  const int q_row = it.row0 + it.qtile * kTileRows;

  if (warp == 0) {
    // ===================================================== producer
    int issued = 0;
    if (lane == 0) {
      tma_prefetch_desc(&tm_q);
      tma_prefetch_desc(&tm_k);
      tma_prefetch_desc(&tm_v);
      mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
#pragma unroll
      for (int a = 0; a < kAtoms; ++a)
        tma_load_2d(sm.q + a * (kTileRows * 128), &tm_q, &sm.q_full, head * D + a * 64, q_row);
    }
    for (int t = 0; t < nkv; ++t) {
      const int st = t % kStages;
      if (t >= kStages) {
        if (!mbar_wait(&sm.kv_empty[st], ((t / kStages) - 1) & 1, abort_flag, g.status)) break;
      }
      const int c0 = it.row0 + kr.tile(t, it.qtile) * kTileRows;
      if (use_time) {
        long long mn = LLONG_MAX, mx = LLONG_MIN;
#pragma unroll
        for (int u = 0; u < kTileRows / 32; ++u) {
          const int c = lane + 32 * u;
          long long tv = 0;
          if (c0 + c < g.T) {
            tv = g.ts[c0 + c];
            mn = tv < mn ? tv : mn;
            mx = tv > mx ? tv : mx;
          }
          sm.ts[st][c] = tv;
        }
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) {
          const long long omn = __shfl_xor_sync(0xffffffffu, mn, off);
          const long long omx = __shfl_xor_sync(0xffffffffu, mx, off);
          mn = omn < mn ? omn : mn;
          mx = omx > mx ? omx : mx;
        }
        if (lane == 0) {
          sm.tmin[st] = mn;
          sm.tmax[st] = mx;
        }
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.kv_full[st], 2 * kTileBytes);
#pragma unroll
        for (int a = 0; a < kAtoms; ++a) {
          tma_load_2d(sm.k[st] + a * (kTileRows * 128), &tm_k, &sm.kv_full[st], head * D + a * 64, c0);
          tma_load_2d(sm.v[st] + a * (kTileRows * 128), &tm_v, &sm.kv_full[st], head * D + a * 64, c0);
        }
      }
      issued = t + 1;
    }
    if (*abort_flag && lane == 0) {
      // leave no TMA write in flight into shared memory that is about to be released
      for (int t = (issued > kStages ? issued - kStages : 0); t < issued; ++t)
        mbar_wait(&sm.kv_full[t % kStages], (t / kStages) & 1, nullptr, nullptr);
      mbar_wait(&sm.q_full, 0, nullptr, nullptr);
    }
  } else if (warp == 1) {
    // ===================================================== MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, 128, 0, 0);
      constexpr uint32_t idesc_o = idesc_bf16_f32(128, D, 0, 1);
      const uint32_t q_base = smem_u32(sm.q);
      bool ok = mbar_wait(&sm.q_full, 0, abort_flag, g.status);
      auto issue_s = [&](int st) {
        const uint32_t k_base = smem_u32(sm.k[st]);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk / 4) * (kTileRows * 128) + (kk % 4) * 32;
          mma_bf16_ss(tmem + kColS, smem_desc_sw128(q_base + off, 16, 1024),
                      smem_desc_sw128(k_base + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
        }
        mma_commit(&sm.s_full);
      };
      if (ok && nkv > 0) {
        ok = mbar_wait(&sm.kv_full[0], 0, abort_flag, g.status);
        if (ok) issue_s(0);
      }
      for (int t = 0; ok && t < nkv; ++t) {
        const int st = t % kStages;
        ok = mbar_wait(&sm.p_full, t & 1, abort_flag, g.status);
        if (!ok) break;
        tc_fence_after();
        const uint32_t v_base = smem_u32(sm.v[st]);
#pragma unroll
        for (int kk = 0; kk < kTileRows / 16; ++kk) {
          mma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8,
                      smem_desc_sw128(v_base + kk * 2048, kTileRows * 128, 1024), idesc_o,
                      (t > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&sm.kv_empty[st]);
        if (t + 1 < nkv) {
          const int st1 = (t + 1) % kStages;
          ok = mbar_wait(&sm.kv_full[st1], ((t + 1) / kStages) & 1, abort_flag, g.status);
          if (!ok) break;
          issue_s(st1);
        }
      }
      mma_commit(&sm.o_full);
      if (!ok) {
        mma_commit(&sm.drain);
        mbar_wait(&sm.drain, 0, nullptr, nullptr);
      }
    }
    __syncwarp();
  } else {
    // ===================================================== epilogue (one thread per row)
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int i = it.qtile * kTileRows + r;  // query index local to the sequence
    const bool row_valid = i < L;
    const int pi = i < n ? i : n;
    const long long ti = (use_time && row_valid) ? g.ts[it.row0 + i] : 0;
    const uint32_t lane_addr = tmem + (static_cast<uint32_t>(quad * 32) << 16);
    const float half_alpha = 0.5f * g.alpha;
    const float* time_tab = sm.rab_time;
    const int32_t* types_seq = g.rab_type != nullptr ? g.types + it.row0 : nullptr;
    const float* type_row =
        g.rab_type != nullptr ? g.rab_type + (row_valid ? types_seq[i] : 0) * g.NT : nullptr;
    bool ok = true;
    for (int t = 0; t < nkv; ++t) {
      const int st = t % kStages;
      const int c0l = kr.tile(t, it.qtile) * kTileRows;
      bool w = !use_time || mbar_wait(&sm.kv_full[st], (t / kStages) & 1, abort_flag, g.status);
      w = w && mbar_wait(&sm.s_full, t & 1, abort_flag, g.status);
      if (!warp_all(w)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // classify this row's segment [c0l, c0l + 128)
      const int last = c0l + kTileRows - 1;
      const bool full_vis = row_valid && last <= i && last < n;
      int mode = 2;
      float half_bias = 0.f;
      if (full_vis) {
        bool uni = type_row == nullptr;  // the token-type term varies along the row
        float bias = 0.f;
        if (pos_tab != nullptr) {
          const int dmin = pi - last;  // smallest position difference in the segment
          if (dmin >= g.P) bias += pos_tab[2 * g.P];
          else uni = false;
        }
        if (use_time && uni) {
          const int b_lo = time_bucket64(ti - sm.tmax[st], g.NB);
          const int b_hi = time_bucket64(ti - sm.tmin[st], g.NB);
          if (b_lo == b_hi) bias += time_tab[b_lo];
          else uni = false;
        }
        mode = uni ? 0 : 1;
        half_bias = 0.5f * bias;
      }
      const long long* ts_tile = sm.ts[st];
#pragma unroll 1
      for (int ch = 0; ch < kTileRows / 32; ++ch) {
        uint32_t s[32];
        uint32_t pk[16];
        tmem_ld32(lane_addr + kColS + ch * 32, s);
        tmem_wait_ld();
        const int cb = c0l + ch * 32;
        if (mode == 0)
          silu_chunk<D, 0>(s, pk, half_alpha, half_bias, cb, i, pi, n, g.P, pos_tab, time_tab,
                           use_time, ts_tile, ti, g.NB, row_valid, types_seq, type_row, L);
        else if (mode == 1)
          silu_chunk<D, 1>(s, pk, half_alpha, half_bias, cb, i, pi, n, g.P, pos_tab, time_tab,
                           use_time, ts_tile, ti, g.NB, row_valid, types_seq, type_row, L);
        else
          silu_chunk<D, 2>(s, pk, half_alpha, half_bias, cb, i, pi, n, g.P, pos_tab, time_tab,
                           use_time, ts_tile, ti, g.NB, row_valid, types_seq, type_row, L);
        tmem_st16(lane_addr + kColP + ch * 16, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full);
    }
    if (ok && warp_all(mbar_wait(&sm.o_full, 0, abort_flag, g.status))) {
      tc_fence_after();
#pragma unroll 1
      for (int ch = 0; ch < D / 32; ++ch) {
        uint32_t o[32];
        tmem_ld32(lane_addr + kColO + ch * 32, o);
        tmem_wait_ld();
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(out + static_cast<int64_t>(it.row0 + i) * ld_o +
                                                head * D + ch * 32);
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            uint4 vv;
            vv.x = pack_bf16x2(__uint_as_float(o[8 * w + 0]), __uint_as_float(o[8 * w + 1]));
            vv.y = pack_bf16x2(__uint_as_float(o[8 * w + 2]), __uint_as_float(o[8 * w + 3]));
            vv.z = pack_bf16x2(__uint_as_float(o[8 * w + 4]), __uint_as_float(o[8 * w + 5]));
            vv.w = pack_bf16x2(__uint_as_float(o[8 * w + 6]), __uint_as_float(o[8 * w + 7]));
            dst[w] = vv;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kAlloc);
  }
}

}  // namespace

template <int D>
static size_t fwd_smem_bytes(int P, bool has_pos) {
  size_t pos = (has_pos && 2 * P + 1 <= kPosSmemMax) ? static_cast<size_t>(2 * P + 1) : 1;
  return sizeof(FwdSmem<D>) + pos * sizeof(float) + 1024;
}

// Launches the tensor-core forward.  Returns a cudaError_t.
cudaError_t launch_attn_fwd_tc(int D, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const AttnGeom& g, __nv_bfloat16* out,
                               int64_t ld_o, int grid, cudaStream_t stream) {
  if (grid <= 0) return cudaSuccess;
  if (D == 64) {
    size_t smem = fwd_smem_bytes<64>(g.P, g.rab_pos != nullptr);
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<64>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_fwd_tc_kernel<64><<<grid, kThreads, smem, stream>>>(tq, tk, tv, g, out, ld_o);
  } else if (D == 128) {
    size_t smem = fwd_smem_bytes<128>(g.P, g.rab_pos != nullptr);
    cudaError_t e = cudaFuncSetAttribute(attn_fwd_tc_kernel<128>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attn_fwd_tc_kernel<128><<<grid, kThreads, smem, stream>>>(tq, tk, tv, g, out, ld_o);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace hstu
