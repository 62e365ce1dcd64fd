// common.cuh — types shared by the kernels and the C-ABI layer.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace hstu {

// Query rows of one attention tile, and key/value rows of one KV tile.
constexpr int kTileRows = 128;

// One unit of attention work: a 128-row query tile of one sequence (all heads share the list).
// len = sequence length, row0 = first token of the sequence, qtile = tile index within it,
// cost = number of KV tiles the tile visits (used only for the longest-first ordering).
struct WorkItem {
  int32_t seq;
  int32_t qtile;
  int32_t row0;
  int32_t len;
};

// Geometry of the jagged problem and bias parameters, passed by value to the kernels.
struct AttnGeom {
  const WorkItem* items;
  const int32_t* item_count;
  const int64_t* ts;        // [T] or nullptr
  const float* rab_pos;     // [2P+1] or nullptr
  const float* rab_time;    // [NB] or nullptr
  int32_t P;
  int32_t NB;
  int32_t H;
  int32_t T;
  int32_t mask;             // 0 causal, 1 M-FALCON
  int32_t num_candidates;
  float alpha;
  int32_t* status;
  // token-type term rab_type[type_i * NT + type_j] (types [T] in [0, NT)), or nullptr
  const int32_t* types;
  const float* rab_type;
  int32_t NT;
  float* d_type;            // backward: gradient of rab_type [NT*NT] (accumulated), or nullptr
  // forward (paired kernel): per output row, the mean and the sum of squared deviations of
  // each 32-column slice of the bf16 output, [T][H d_v / 32] float2, or nullptr (the
  // LayerNorm statistics of the layer's output projection, combined there)
  float2* o_stats;
};

// One launch of the persistent tensor-core GEMM (gemm_tc.cu): C[M, N] = epi(A · B), A and B
// through the tensor maps ta / tb in the layouts a_mn / b_mn select; see the kernel's comment.
struct GemmArgs {
  const CUtensorMap* ta;
  const CUtensorMap* tb;
  const CUtensorMap* tc;           // epi 0-3: C, box {32, 32}, 64-byte swizzle (TMA store)
  const CUtensorMap* tr;           // epi 1: the residual, same box and swizzle
  int M, N, K, k_splits;
  int epi, a_mn, b_mn;
  const float* bias;               // [N] or nullptr
  const __nv_bfloat16* resid;      // epi 1
  int64_t ld_r;
  __nv_bfloat16* C;                // epi 0-3
  int64_t ldc;                     // row stride of C (or of Cf for epi 4)
  float* C2;                       // epi 3: the pre-activation (fp32)
  int64_t ld_c2;
  float* Cf;                       // epi 4: fp32 [M, N], accumulated into
  int* status;
};

// SiLU' factors for a backward that produces dpre = dA ⊙ SiLU'(Z) directly: fp32 pre-activation
// columns of the Q, K, V (and U) blocks, row stride ld (elements); q == nullptr: none.
struct SiluGradZ {
  const float* q;
  const float* k;
  const float* v;
  int64_t ld;
};

// SiLU'(z) = σ(z) (1 + z (1 - σ(z))), σ(z) = (1 + tanh(z / 2)) / 2.
__device__ __forceinline__ float silu_grad_z(float z) {
  float t;
  asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * z));
  const float sg = fmaf(0.5f, t, 0.5f);
  return sg * fmaf(z, 1.f - sg, 1.f);
}

// History length n of a sequence: every token for the causal mask, L - m under M-FALCON.
__host__ __device__ __forceinline__ int hist_len(int L, int mask, int m) {
  if (mask == 1) {
    int n = L - m;
    return n < 0 ? 0 : n;
  }
  return L;
}

// KV tiles a query tile visits: tiles 0 .. nh-1 cover every key j < min(qe, n) (the visible
// history), plus the query tile's own diagonal tile when it holds candidates that only see
// themselves beyond the history.  Causal: nh = qtile + 1 and no extra tile.
struct KvRange {
  int nh;
  int diag;  // 1 if the diagonal tile is visited after the nh history tiles
  __device__ __forceinline__ int count() const { return nh + diag; }
  __device__ __forceinline__ int tile(int t, int qtile) const { return t < nh ? t : qtile; }
};

__device__ __forceinline__ KvRange kv_range(int qtile, int L, int n) {
  const int qs = qtile * kTileRows;
  const int qe = min(qs + kTileRows, L);
  const int hv = min(qe, n);
  KvRange r;
  r.nh = (hv + kTileRows - 1) / kTileRows;
  r.diag = (qe > n && qtile >= r.nh) ? 1 : 0;
  return r;
}

}  // namespace hstu
