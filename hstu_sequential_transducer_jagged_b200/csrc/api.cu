// api.cu — the C ABI declared in include/hstu.h: host-side argument checks, workspace layout,
// TMA tensor-map encoding, and kernel dispatch on the caller's stream.  No device memory is
// allocated here and nothing synchronises with the device except hstu_sync_status().
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/hstu.h"
#include "common.cuh"

namespace hstu {
cudaError_t launch_attn_fwd_tc(int D, const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const AttnGeom& g, __nv_bfloat16* out,
                               int64_t ld_o, int grid, cudaStream_t stream);
cudaError_t launch_gemm_tc(const GemmArgs& a, cudaStream_t stream);
int gemm_tc_mn_tiles(int M, int N);
cudaError_t launch_build_worklist(const int32_t* offsets, int B, int T, int max_len, int mask,
                                  int m, int group, int cand_only, WorkItem* items,
                                  int32_t* count, int32_t* hist, int max_cost, int32_t* status,
                                  cudaStream_t stream);
cudaError_t launch_attn_fwd_pair(const CUtensorMap& tq, const CUtensorMap& tk,
                                 const CUtensorMap& tv, const CUtensorMap& tts,
                                 const AttnGeom& g, __nv_bfloat16* out, int64_t ld_o, int grid,
                                 cudaStream_t stream);
size_t attn_fwd_pair_smem(int P, bool has_pos);
int attn_fwd_pair_kv_rows();
int attn_fwd_pair_ts_box();
cudaError_t launch_ln_gate(int dtype, const void* av, int64_t ld_av, const void* u, int64_t ld_u,
                           const float* gamma, const float* beta, float eps, void* g,
                           int64_t ld_g, int rows, int F, cudaStream_t stream);
cudaError_t launch_jagged_padded(const int32_t* offsets, int B, int max_len, const void* jag,
                                 int64_t jag_stride, void* pad, int64_t pad_stride,
                                 int64_t row_bytes, int to_padded, int num_sms,
                                 cudaStream_t stream);
cudaError_t launch_time_buckets(const int64_t* dt, int n, int32_t* out, int nb,
                                cudaStream_t stream);
cudaError_t launch_bias_index(int rule, const int64_t* in, int n, int param, int32_t* out,
                              cudaStream_t stream);
cudaError_t launch_wait_timeout_probe(int32_t* status, cudaStream_t stream);
cudaError_t launch_attn_fwd_simt(int dtype, int D, const AttnGeom& g, const void* q, int64_t ld_q,
                                 const void* k, int64_t ld_k, const void* v, int64_t ld_v,
                                 void* o, int64_t ld_o, int grid, cudaStream_t stream);
cudaError_t launch_gemm_simt(int dtype, int epi, const void* A, int64_t lda, const void* B,
                             int64_t ldb, int M, int N, int K, const float* bias, const void* R,
                             int64_t ldr, void* C, int64_t ldc, cudaStream_t stream);
cudaError_t launch_attn_bwd_simt(int dtype, int D, const AttnGeom& g, const void* q, int64_t ld_q,
                                 const void* k, int64_t ld_k, const void* v, int64_t ld_v,
                                 const void* d_o, int64_t ld_do, void* dq, void* dk, void* dv,
                                 float* d_pos, float* d_time, int grid, cudaStream_t stream);
cudaError_t launch_attn_bwd_tc(const CUtensorMap& tq, const CUtensorMap& tk,
                               const CUtensorMap& tv, const CUtensorMap& tdo,
                               const CUtensorMap& tts, const CUtensorMap& tdq, const AttnGeom& g, __nv_bfloat16* dq,
                               int64_t ld_dq, __nv_bfloat16* dk, int64_t ld_dk,
                               __nv_bfloat16* dv, int64_t ld_dv, float* dq_acc, float* d_pos,
                               float* d_time, int grid, bool fast, const SiluGradZ& zg,
                               cudaStream_t stream);
size_t attn_bwd_tc_smem(int P, int NB);
cudaError_t launch_ln_gate_bwd(const __nv_bfloat16* av, int64_t ld_av, const __nv_bfloat16* u,
                               int64_t ld_u, const __nv_bfloat16* dg, int64_t ld_dg,
                               const float* gamma, const float* beta, float eps,
                               __nv_bfloat16* d_av, int64_t ld_dav, __nv_bfloat16* d_u,
                               int64_t ld_du, const float* z_u, int64_t ld_z, float* d_gamma,
                               float* d_beta, int rows, int F, int num_sms,
                               cudaStream_t stream);
cudaError_t launch_silu_grad_mul(const float* z, int64_t ld_z, const __nv_bfloat16* da,
                                 int64_t ld_da, __nv_bfloat16* dz, int64_t ld_dz, int rows,
                                 int cols, int num_sms, cudaStream_t stream);
cudaError_t launch_stochastic_length(const int32_t* off, int B, int T, int max_len, int sub_len,
                                     double n_alpha, const float* u, const uint32_t* keys,
                                     int32_t* local_idx, int32_t* lens, int32_t* new_off,
                                     int32_t* kept, int32_t* status, cudaStream_t stream);
cudaError_t launch_gather_rows(const void* src, int64_t src_stride, const int32_t* index,
                               const int32_t* count, int n, void* dst, int64_t dst_stride,
                               int64_t row_bytes, int num_sms, cudaStream_t stream);
cudaError_t launch_candidate_rows(const int32_t* off, int B, int m, int32_t* idx, int32_t* status,
                                  cudaStream_t stream);
cudaError_t launch_scatter_rows(const void* src, int64_t src_stride, const int32_t* index, int n,
                                void* dst, int64_t dst_stride, int64_t row_bytes, int num_sms,
                                cudaStream_t stream);
bool f2_fused_supported(int F, int N);
cudaError_t launch_f2_fused(const CUtensorMap& tm_av, const CUtensorMap& tm_u,
                            const CUtensorMap& tm_w2, const CUtensorMap& tm_x,
                            const CUtensorMap& tm_y, const __nv_bfloat16* av, int64_t ld_av,
                            int M, int N, int F, const float* gamma, const float* beta, float eps,
                            const float* bias, float2* stats, int nparts, int* status,
                            int num_sms, cudaStream_t stream);
cudaError_t launch_colsum(const __nv_bfloat16* m, int64_t ld, int rows, int cols, float* out,
                          cudaStream_t stream);
int attn_bwd_tc_ts_box();
}  // namespace hstu

using namespace hstu;

namespace {

thread_local char g_last_error[256] = "";

// Records a CUDA error's text for hstu_last_error_string() and maps it to HSTU_ERR_CUDA.
hstu_status_t cuda_fail(cudaError_t e) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", cudaGetErrorName(e),
                cudaGetErrorString(e));
  return HSTU_ERR_CUDA;
}

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;  // status word at 0, work-item count at 4
constexpr int kMaxSeqLen = 1 << 24;
// Largest position clamp P: 2P + 1 table entries and every index stay far inside int32.
constexpr int kMaxPosDist = 1 << 24;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// ----------------------------------------------------------------- driver entry points
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

int num_sms_current() {
  int dev = 0, n = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

// 2D bf16 tensor map over a row-major [rows, cols] matrix with row stride ld (elements), box
// {box_cols, box_rows}, the given swizzle, zero fill out of bounds.
bool make_map_bf16_sw(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                      uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The same with 128-byte swizzle (the MMA operand tiles).
bool make_map_bf16(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                   uint32_t box_cols, uint32_t box_rows) {
  return make_map_bf16_sw(map, base, rows, cols, ld, box_cols, box_rows,
                          CU_TENSOR_MAP_SWIZZLE_128B);
}

// Maps of a GEMM's bf16 output C and residual R for the staged TMA epilogue: 32 x 32 boxes,
// 64-byte swizzle.  Absent matrices get zeroed (unused) maps.
bool make_epilogue_maps(CUtensorMap* tc, CUtensorMap* tr, const void* C, int64_t ldc,
                        const void* R, int64_t ldr, int M, int N) {
  std::memset(tc, 0, sizeof(*tc));
  std::memset(tr, 0, sizeof(*tr));
  if (C != nullptr && !make_map_bf16_sw(tc, C, M, N, ldc, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return false;
  if (R != nullptr && !make_map_bf16_sw(tr, R, M, N, ldr, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return false;
  return true;
}

// 2D fp32 tensor map over a row-major [rows, cols] matrix with row stride ld (elements), box
// {box_cols, box_rows}, 64-byte swizzle (the attention backward's dQ reduction target: 16 x 32
// boxes).
bool make_map_f32(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                  uint32_t box_cols, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

// 1D int64 tensor map over n elements, box of `box` elements, no swizzle, zero fill.
bool make_map_i64_1d(CUtensorMap* map, const void* base, int64_t n, uint32_t box) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[1] = {static_cast<cuuint64_t>(n)};
  cuuint64_t strides[1] = {8};
  cuuint32_t boxd[1] = {box};
  cuuint32_t estr[1] = {1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_INT64, 1, const_cast<void*>(base), dims, strides,
                  boxd, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t elem_size(int dtype) { return dtype == HSTU_BF16 ? 2 : 4; }

// Work-list sizes for a batch: an upper bound of the number of 128-row query tiles
// (Σ ceil(L_b / 128) <= T / 128 + B) and of the cost histogram.
int max_items(int T, int B, int group = 1) {
  return (T + kTileRows * group - 1) / (kTileRows * group) + B;
}
int max_cost(int max_len) { return 2 * ((max_len + kTileRows - 1) / kTileRows + 1); }

struct WsLayout {
  size_t items, hist, total_attn;
};

WsLayout attn_layout(int T, int B, int max_len) {
  WsLayout w;
  w.items = kStatusBytes;
  w.hist = w.items + align_up(sizeof(WorkItem) * static_cast<size_t>(max_items(T, B)));
  w.total_attn = w.hist + align_up(sizeof(int32_t) * static_cast<size_t>(max_cost(max_len) + 1));
  return w;
}

hstu_status_t check_common(int B, int T, int max_len, const int32_t* offsets, int H, int dqk,
                           int dv, int mask, int m, int mb, const float* rab_pos, int P,
                           const float* rab_time, int NB, float alpha, int dtype) {
  if (B < 0 || T < 0 || max_len < 0 || max_len > kMaxSeqLen) return HSTU_ERR_INVALID_ARG;
  if (B > 0 && offsets == nullptr) return HSTU_ERR_INVALID_ARG;
  if (H < 1 || dqk < 1 || dv < 1) return HSTU_ERR_INVALID_ARG;
  if (mask != HSTU_MASK_CAUSAL && mask != HSTU_MASK_MFALCON) return HSTU_ERR_INVALID_ARG;
  if (mask == HSTU_MASK_MFALCON && (m < 0 || mb < 1)) return HSTU_ERR_INVALID_ARG;
  if (rab_pos != nullptr && (P < 0 || P > kMaxPosDist)) return HSTU_ERR_INVALID_ARG;
  if (rab_time != nullptr && NB < 1) return HSTU_ERR_INVALID_ARG;
  if (!std::isfinite(alpha)) return HSTU_ERR_INVALID_ARG;
  if (dtype != HSTU_BF16 && dtype != HSTU_FP32) return HSTU_ERR_INVALID_ARG;
  if (static_cast<int64_t>(max_len) * 1 > 0 && T > 0 && static_cast<int64_t>(B) * max_len < T)
    return HSTU_ERR_INVALID_ARG;  // max_len too small to hold T tokens in B sequences
  if (dqk != dv) return HSTU_ERR_UNSUPPORTED;
  if (dqk != 16 && dqk != 32 && dqk != 64 && dqk != 128) return HSTU_ERR_UNSUPPORTED;
  return HSTU_OK;
}

hstu_status_t check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0 || ws_bytes < need)
    return HSTU_ERR_WORKSPACE;
  return HSTU_OK;
}

AttnGeom make_geom(const void* ws, const WsLayout& w, const int64_t* ts, const float* rab_pos,
                   int P, const float* rab_time, int NB, int H, int T, int mask, int m,
                   float alpha) {
  uint8_t* base = static_cast<uint8_t*>(const_cast<void*>(ws));
  AttnGeom g;
  g.items = reinterpret_cast<const WorkItem*>(base + w.items);
  g.item_count = reinterpret_cast<const int32_t*>(base + 4);
  g.ts = ts;
  g.rab_pos = rab_pos;
  g.rab_time = rab_time;
  g.P = P;
  g.NB = NB;
  g.H = H;
  g.T = T;
  g.mask = mask;
  g.num_candidates = (mask == HSTU_MASK_MFALCON) ? m : 0;
  g.alpha = alpha;
  g.status = reinterpret_cast<int32_t*>(base);
  g.types = nullptr;
  g.rab_type = nullptr;
  g.NT = 0;
  g.d_type = nullptr;
  g.o_stats = nullptr;
  return g;
}

// The token-type term's arguments (rab_type NULL: off).
hstu_status_t check_types(const int32_t* types, const float* rab_type, int NT, int T) {
  if (rab_type == nullptr) return HSTU_OK;
  if (NT < 1 || NT > 64 || (T > 0 && types == nullptr)) return HSTU_ERR_INVALID_ARG;
  return HSTU_OK;
}

void set_types(AttnGeom* g, const int32_t* types, const float* rab_type, int NT) {
  if (rab_type == nullptr) return;
  g->types = types;
  g->rab_type = rab_type;
  g->NT = NT;
}

cudaError_t build_list(const void* ws, const WsLayout& w, const int32_t* offsets, int B, int T,
                       int max_len, int mask, int m, int group, cudaStream_t s,
                       int cand_only = 0) {
  uint8_t* base = static_cast<uint8_t*>(const_cast<void*>(ws));
  return launch_build_worklist(offsets, B, T, max_len, mask, mask == HSTU_MASK_MFALCON ? m : 0,
                               group, cand_only,
                               reinterpret_cast<WorkItem*>(base + w.items),
                               reinterpret_cast<int32_t*>(base + 4),
                               reinterpret_cast<int32_t*>(base + w.hist), max_cost(max_len),
                               reinterpret_cast<int32_t*>(base), s);
}

// True when the tensor-core kernels take this attention problem.
bool attn_uses_tc(int D, int dtype, const void* q, int64_t ld_q, const void* k, int64_t ld_k,
                  const void* v, int64_t ld_v, const void* o, int64_t ld_o) {
  return dtype == HSTU_BF16 && (D == 64 || D == 128) && aligned16(q) && aligned16(k) &&
         aligned16(v) && aligned16(o) && (ld_q % 8 == 0) && (ld_k % 8 == 0) && (ld_v % 8 == 0) &&
         (ld_o % 8 == 0);
}

// The paired kernel: bf16 tensor cores, head dimension 64, no type term; it keeps the position
// table in shared memory (it fits for P up to about 1100 next to its tiles: the shared-memory
// check decides) and loads the timestamps with TMA (16-byte aligned base).
bool attn_uses_pair(const AttnGeom& g, int D, bool tc) {
  const bool use_time = g.ts != nullptr && g.rab_time != nullptr;
  return tc && D == 64 && g.rab_type == nullptr && (g.rab_pos == nullptr || g.P <= 2048) &&
         (!use_time || aligned16(g.ts)) &&
         attn_fwd_pair_smem(g.P, g.rab_pos != nullptr) <= 227 * 1024;
}

// Builds the work list (pairs of query tiles for the head-width-64 tensor-core kernel, single
// tiles otherwise) and launches the attention forward.
hstu_status_t attn_forward_core(const void* ws, const WsLayout& w, const int32_t* offsets,
                                int max_len, const AttnGeom& g, int B, int T, int D, int dtype,
                                const void* q, int64_t ld_q, const void* k, int64_t ld_k,
                                const void* v, int64_t ld_v, void* o, int64_t ld_o,
                                cudaStream_t s, int cand_only = 0) {
  const bool tc = attn_uses_tc(D, dtype, q, ld_q, k, ld_k, v, ld_v, o, ld_o);
  const bool use_time = g.ts != nullptr && g.rab_time != nullptr;
  const bool pair = attn_uses_pair(g, D, tc);
  const int group = pair ? 2 : 1;
  if (build_list(ws, w, offsets, B, T, max_len, g.mask, g.num_candidates, group, s, cand_only) !=
      cudaSuccess)
    return HSTU_ERR_CUDA;
  const int grid = max_items(T, B, group) * g.H;
  cudaError_t e;
  if (tc) {
    CUtensorMap tq, tk, tv;
    const int64_t cols = static_cast<int64_t>(g.H) * D;
    // the paired kernel streams K / V in shorter tiles than its query tiles
    const uint32_t kv_rows = pair ? static_cast<uint32_t>(attn_fwd_pair_kv_rows()) : kTileRows;
    if (!make_map_bf16(&tq, q, T, cols, ld_q, 64, kTileRows) ||
        !make_map_bf16(&tk, k, T, cols, ld_k, 64, kv_rows) ||
        !make_map_bf16(&tv, v, T, cols, ld_v, 64, kv_rows))
      return HSTU_ERR_CUDA;
    if (pair) {
      CUtensorMap tts;
      std::memset(&tts, 0, sizeof(tts));
      if (use_time && !make_map_i64_1d(&tts, g.ts, T, attn_fwd_pair_ts_box()))
        return HSTU_ERR_CUDA;
      // persistent: one CTA per SM, each walking the work list with a stride
      const int pgrid = grid < num_sms_current() ? grid : num_sms_current();
      e = launch_attn_fwd_pair(tq, tk, tv, tts, g, static_cast<__nv_bfloat16*>(o), ld_o, pgrid,
                               s);
    }
    else
      e = launch_attn_fwd_tc(D, tq, tk, tv, g, static_cast<__nv_bfloat16*>(o), ld_o, grid, s);
  } else {
    e = launch_attn_fwd_simt(dtype, D, g, q, ld_q, k, ld_k, v, ld_v, o, ld_o, grid, s);
  }
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

// C = epi(A[M,K] B[K,N] + bias) on tensor cores when the shapes allow, else on CUDA cores.
hstu_status_t gemm(int dtype, int epi, const void* A, int64_t lda, const void* Bm, int64_t ldb,
                   int M, int N, int K, const float* bias, const void* R, int64_t ldr, void* C,
                   int64_t ldc, int32_t* status, cudaStream_t s) {
  const bool tc = dtype == HSTU_BF16 && K % 8 == 0 && N % 8 == 0 && lda % 8 == 0 &&
                  ldb % 8 == 0 && ldc % 8 == 0 && (R == nullptr || ldr % 8 == 0) &&
                  aligned16(A) && aligned16(Bm) && aligned16(C) && (R == nullptr || aligned16(R));
  cudaError_t e;
  if (tc) {
    CUtensorMap ta, tb, tcm, trm;
    if (!make_map_bf16(&ta, A, M, K, lda, 64, 128) || !make_map_bf16(&tb, Bm, K, N, ldb, 64, 64) ||
        !make_epilogue_maps(&tcm, &trm, C, ldc, R, ldr, M, N))
      return HSTU_ERR_CUDA;
    GemmArgs ga{};
    ga.ta = &ta;
    ga.tb = &tb;
    ga.tc = &tcm;
    ga.tr = &trm;
    ga.M = M;
    ga.N = N;
    ga.K = K;
    ga.k_splits = 1;
    ga.epi = epi;
    ga.a_mn = 0;
    ga.b_mn = 1;
    ga.bias = bias;
    ga.resid = static_cast<const __nv_bfloat16*>(R);
    ga.ld_r = ldr;
    ga.C = static_cast<__nv_bfloat16*>(C);
    ga.ldc = ldc;
    ga.status = status;
    e = launch_gemm_tc(ga, s);
  } else {
    e = launch_gemm_simt(dtype, epi, A, lda, Bm, ldb, M, N, K, bias, R, ldr, C, ldc, s);
  }
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

// Y = X + (Norm(AV) ⊙ U) W2 + b2 over `rows` tokens: for bf16 with H d_v <= 1024 a row-statistics
// pass and one fused tensor-core kernel (G formed in shared memory), else LayerNorm ⊙ U into
// g_buf and the GEMM.
bool norm_gate_f2_fused(int dtype, const void* av, int64_t ld_av, const void* u, int64_t ld_u,
                        const void* w2, const void* x, const void* y, int F, int d_model) {
  return dtype == HSTU_BF16 && f2_fused_supported(F, d_model) && ld_av % 8 == 0 &&
         ld_u % 8 == 0 && d_model % 8 == 0 && aligned16(av) && aligned16(u) && aligned16(w2) &&
         aligned16(x) && aligned16(y);
}

// nparts > 0: g_buf already holds the attention kernel's per-slice statistics of av (F / 32
// slices a row); else the fused path computes them into g_buf first.
hstu_status_t norm_gate_f2(int dtype, const void* av, int64_t ld_av, const void* u, int64_t ld_u,
                           const float* gamma, const float* beta, float eps, const void* w2,
                           const float* b2, const void* x, void* y, int rows, int F, int d_model,
                           void* g_buf, int32_t* status, cudaStream_t s, int nparts = 0) {
  if (norm_gate_f2_fused(dtype, av, ld_av, u, ld_u, w2, x, y, F, d_model)) {
    CUtensorMap tav, tu, tw2, ty, tx;
    if (!make_map_bf16(&tav, av, rows, F, ld_av, 64, 128) ||
        !make_map_bf16(&tu, u, rows, F, ld_u, 64, 128) ||
        !make_map_bf16(&tw2, w2, F, d_model, d_model, 64, 64) ||
        !make_epilogue_maps(&ty, &tx, y, d_model, x, d_model, rows, d_model))
      return HSTU_ERR_CUDA;
    // g_buf (rows x F elements) holds the per-row (mean, rstd) pairs instead of G
    const cudaError_t e = launch_f2_fused(
        tav, tu, tw2, tx, ty, static_cast<const __nv_bfloat16*>(av), ld_av, rows, d_model, F,
        gamma, beta, eps, b2, static_cast<float2*>(g_buf), nparts, status, num_sms_current(), s);
    return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
  }
  if (launch_ln_gate(dtype == HSTU_BF16 ? 0 : 1, av, ld_av, u, ld_u, gamma, beta, eps, g_buf, F,
                     rows, F, s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  return gemm(dtype, 1, g_buf, F, w2, d_model, rows, d_model, F, b2, x, d_model, y, d_model,
              status, s);
}

// C = epi(op(A) op(B)) on the tensor cores for the backward's operand layouts: a_mn = 1 takes A
// stored [K, M] (lda its row stride), b_mn = 0 takes B stored [N, K].  epi 3 also writes the
// fp32 pre-activation to C2; epi 4 accumulates fp32 into Cf with k_splits work units per tile.
hstu_status_t gemm_tc_layout(int epi, int a_mn, int b_mn, const void* A, int64_t lda,
                             const void* Bm, int64_t ldb, int M, int N, int K, int k_splits,
                             const float* bias, const void* R, int64_t ldr, void* C, int64_t ldc, void* C2,
                             int64_t ld_c2, float* Cf, int32_t* status, cudaStream_t s) {
  CUtensorMap ta, tb;
  const bool ok_a = a_mn ? make_map_bf16(&ta, A, K, M, lda, 64, 64)
                         : make_map_bf16(&ta, A, M, K, lda, 64, 128);
  const bool ok_b = b_mn ? make_map_bf16(&tb, Bm, K, N, ldb, 64, 64)
                         : make_map_bf16(&tb, Bm, N, K, ldb, 64, 256);
  CUtensorMap tcm, trm;
  if (!ok_a || !ok_b ||
      !make_epilogue_maps(&tcm, &trm, epi == 4 ? nullptr : C, ldc, epi == 1 ? R : nullptr, ldr, M,
                          N))
    return HSTU_ERR_CUDA;
  GemmArgs ga{};
  ga.ta = &ta;
  ga.tb = &tb;
  ga.tc = &tcm;
  ga.tr = &trm;
  ga.M = M;
  ga.N = N;
  ga.K = K;
  ga.k_splits = k_splits;
  ga.epi = epi;
  ga.a_mn = a_mn;
  ga.b_mn = b_mn;
  ga.bias = bias;
  ga.resid = static_cast<const __nv_bfloat16*>(R);
  ga.ld_r = ldr;
  ga.C = static_cast<__nv_bfloat16*>(C);
  ga.ldc = ldc;
  ga.C2 = static_cast<float*>(C2);
  ga.ld_c2 = ld_c2;
  ga.Cf = Cf;
  ga.status = status;
  const cudaError_t e = launch_gemm_tc(ga, s);
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

// Split-K factor that gives about one work unit per SM for an M x N fp32 weight gradient.
int weight_grad_splits(int M, int N, int K) {
  const int tiles = gemm_tc_mn_tiles(M, N);
  const int kblocks = (K + 63) / 64;
  int ks = num_sms_current() / (tiles > 0 ? tiles : 1);
  if (ks < 1) ks = 1;
  if (ks > kblocks) ks = kblocks > 0 ? kblocks : 1;
  return ks;
}

// Layout of the layer backward's workspace: the attention backward's (status word, work list,
// fp32 dQ accumulator) first, then the saved and gradient activations.
struct LayerBwdLayout {
  size_t attn, z, a, av, g, dg, dav, da, total;
};

LayerBwdLayout layer_bwd_layout(const hstu_layer_desc_t* d, const hstu_attn_desc_t& ad) {
  const size_t T = static_cast<size_t>(d->total_tokens);
  const size_t n1 = 2 * static_cast<size_t>(d->num_heads) * (d->d_qk + d->d_v);
  const size_t hv = static_cast<size_t>(d->num_heads) * d->d_v;
  LayerBwdLayout l;
  l.attn = 0;
  l.z = align_up(hstu_attention_backward_workspace_size(&ad));
  l.a = l.z + align_up(T * n1 * 4);  // the pre-activation in fp32
  l.av = l.a + align_up(T * n1 * 2);
  l.g = l.av + align_up(T * hv * 2);
  l.dg = l.g + align_up(T * hv * 2);
  l.dav = l.dg + align_up(T * hv * 2);
  l.da = l.dav + align_up(T * hv * 2);
  l.total = l.da + align_up(T * n1 * 2);
  return l;
}

// The attention problem of a layer: Q, K, V are column blocks of the f1 output [U | V | Q | K].
hstu_attn_desc_t layer_attn_desc(const hstu_layer_desc_t* d) {
  hstu_attn_desc_t a;
  std::memset(&a, 0, sizeof(a));
  const int64_t n1 = 2 * static_cast<int64_t>(d->num_heads) * (d->d_qk + d->d_v);
  a.num_seqs = d->num_seqs;
  a.total_tokens = d->total_tokens;
  a.max_seq_len = d->max_seq_len;
  a.seq_offsets = d->seq_offsets;
  a.timestamps = d->timestamps;
  a.num_heads = d->num_heads;
  a.d_qk = d->d_qk;
  a.d_v = d->d_v;
  a.ld_q = a.ld_k = a.ld_v = n1;
  a.ld_o = static_cast<int64_t>(d->num_heads) * d->d_v;
  a.mask = d->mask;
  a.num_candidates = d->num_candidates;
  a.mfalcon_microbatch = d->mfalcon_microbatch;
  a.rab_pos = d->rab_pos;
  a.max_pos_dist = d->max_pos_dist;
  a.rab_time = d->rab_time;
  a.num_time_buckets = d->num_time_buckets;
  a.alpha = d->alpha;
  a.dtype = d->dtype;
  a.token_types = d->token_types;
  a.rab_type = d->rab_type;
  a.num_types = d->num_types;
  return a;
}

}  // namespace

namespace {
hstu_status_t attn_backward_impl(const hstu_attn_desc_t* d, const void* q, const void* k,
                                 const void* v, const void* d_o, void* dq, void* dk, void* dv,
                                 float* d_rab_pos, float* d_rab_time, float* d_rab_type,
                                 void* ws, size_t ws_bytes, hstu_stream_t stream,
                                 const SiluGradZ& zg, bool* zg_applied);
}  // namespace

extern "C" {

size_t hstu_attention_workspace_size(const hstu_attn_desc_t* d) {
  if (d == nullptr || d->total_tokens < 0 || d->num_seqs < 0 || d->max_seq_len < 0) return 0;
  return attn_layout(d->total_tokens, d->num_seqs, d->max_seq_len).total_attn;
}

size_t hstu_attention_backward_workspace_size(const hstu_attn_desc_t* d) {
  if (d == nullptr || d->total_tokens < 0 || d->num_seqs < 0 || d->max_seq_len < 0 ||
      d->num_heads < 1 || d->d_qk < 1)
    return 0;
  // + the fp32 dQ accumulator [T, H * d_qk] of the tensor-core backward
  return hstu_attention_workspace_size(d) +
         align_up(sizeof(float) * static_cast<size_t>(d->total_tokens) * d->num_heads * d->d_qk);
}

hstu_status_t hstu_attention_forward(const hstu_attn_desc_t* d, const void* q, const void* k,
                                     const void* v, void* o, void* ws, size_t ws_bytes,
                                     hstu_stream_t stream) {
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  hstu_status_t st = check_common(d->num_seqs, d->total_tokens, d->max_seq_len, d->seq_offsets,
                                  d->num_heads, d->d_qk, d->d_v, d->mask, d->num_candidates,
                                  d->mfalcon_microbatch, d->rab_pos, d->max_pos_dist,
                                  d->rab_time, d->num_time_buckets, d->alpha, d->dtype);
  if (st != HSTU_OK) return st;
  st = check_types(d->token_types, d->rab_type, d->num_types, d->total_tokens);
  if (st != HSTU_OK) return st;
  const int D = d->d_qk;
  const int64_t cols = static_cast<int64_t>(d->num_heads) * D;
  // (row strides mean nothing for an empty batch: views of zero rows may report any stride)
  if (d->total_tokens > 0 &&
      (d->ld_q < cols || d->ld_k < cols || d->ld_v < cols || d->ld_o < cols))
    return HSTU_ERR_INVALID_ARG;
  const WsLayout w = attn_layout(d->total_tokens, d->num_seqs, d->max_seq_len);
  st = check_ws(ws, ws_bytes, w.total_attn);
  if (st != HSTU_OK) return st;
  if (d->num_seqs == 0 || d->total_tokens == 0) return HSTU_OK;
  if (q == nullptr || k == nullptr || v == nullptr || o == nullptr) return HSTU_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  AttnGeom g = make_geom(ws, w, d->timestamps, d->rab_pos, d->max_pos_dist, d->rab_time,
                         d->num_time_buckets, d->num_heads, d->total_tokens, d->mask,
                         d->num_candidates, d->alpha);
  set_types(&g, d->token_types, d->rab_type, d->num_types);
  return attn_forward_core(ws, w, d->seq_offsets, d->max_seq_len, g, d->num_seqs,
                           d->total_tokens, D, d->dtype, q, d->ld_q, k, d->ld_k, v, d->ld_v, o,
                           d->ld_o, s);
}

hstu_status_t hstu_attention_backward(const hstu_attn_desc_t* d, const void* q, const void* k,
                                      const void* v, const void* d_o, void* dq, void* dk,
                                      void* dv, float* d_rab_pos, float* d_rab_time, void* ws,
                                      size_t ws_bytes, hstu_stream_t stream) {
  if (d == nullptr || d->rab_type != nullptr) return HSTU_ERR_INVALID_ARG;
  return hstu_attention_backward_typed(d, q, k, v, d_o, dq, dk, dv, d_rab_pos, d_rab_time,
                                       nullptr, ws, ws_bytes, stream);
}

hstu_status_t hstu_attention_backward_typed(const hstu_attn_desc_t* d, const void* q,
                                            const void* k, const void* v, const void* d_o,
                                            void* dq, void* dk, void* dv, float* d_rab_pos,
                                            float* d_rab_time, float* d_rab_type, void* ws,
                                            size_t ws_bytes, hstu_stream_t stream) {
  return attn_backward_impl(d, q, k, v, d_o, dq, dk, dv, d_rab_pos, d_rab_time, d_rab_type, ws,
                            ws_bytes, stream, SiluGradZ{nullptr, nullptr, nullptr, 0}, nullptr);
}

}  // extern "C"

namespace {
// The attention backward.  zg (a layer's backward) multiplies dQ, dK, dV by SiLU'(Z) before
// their rounding when the tensor-core kernel runs; *zg_applied reports whether it did (the
// CUDA-core kernels leave dQ, dK, dV unscaled).
hstu_status_t attn_backward_impl(const hstu_attn_desc_t* d, const void* q, const void* k,
                                 const void* v, const void* d_o, void* dq, void* dk, void* dv,
                                 float* d_rab_pos, float* d_rab_time, float* d_rab_type,
                                 void* ws, size_t ws_bytes, hstu_stream_t stream,
                                 const SiluGradZ& zg, bool* zg_applied) {
  if (zg_applied != nullptr) *zg_applied = false;
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  {
    const hstu_status_t tst = check_types(d->token_types, d->rab_type, d->num_types,
                                          d->total_tokens);
    if (tst != HSTU_OK) return tst;
    if (d->rab_type != nullptr && d_rab_type == nullptr) return HSTU_ERR_INVALID_ARG;
  }
  hstu_status_t st = check_common(d->num_seqs, d->total_tokens, d->max_seq_len, d->seq_offsets,
                                  d->num_heads, d->d_qk, d->d_v, d->mask, d->num_candidates,
                                  d->mfalcon_microbatch, d->rab_pos, d->max_pos_dist,
                                  d->rab_time, d->num_time_buckets, d->alpha, d->dtype);
  if (st != HSTU_OK) return st;
  const int D = d->d_qk;
  const int64_t cols = static_cast<int64_t>(d->num_heads) * D;
  // (row strides mean nothing for an empty batch: views of zero rows may report any stride)
  if (d->total_tokens > 0 &&
      (d->ld_q < cols || d->ld_k < cols || d->ld_v < cols || d->ld_o < cols))
    return HSTU_ERR_INVALID_ARG;
  if (d->rab_pos != nullptr && d_rab_pos == nullptr) return HSTU_ERR_INVALID_ARG;
  if (d->rab_time != nullptr && d->timestamps != nullptr && d_rab_time == nullptr)
    return HSTU_ERR_INVALID_ARG;
  if (d->rab_pos != nullptr && 2 * static_cast<int64_t>(d->max_pos_dist) + 1 + d->num_time_buckets > 50000)
    return HSTU_ERR_UNSUPPORTED;  // the per-CTA bias-gradient bins live in shared memory
  const WsLayout w = attn_layout(d->total_tokens, d->num_seqs, d->max_seq_len);
  st = check_ws(ws, ws_bytes, hstu_attention_backward_workspace_size(d));
  if (st != HSTU_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (d_rab_pos != nullptr && d->rab_pos != nullptr &&
      cudaMemsetAsync(d_rab_pos, 0, sizeof(float) * (2 * d->max_pos_dist + 1), s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (d_rab_time != nullptr && d->rab_time != nullptr &&
      cudaMemsetAsync(d_rab_time, 0, sizeof(float) * d->num_time_buckets, s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (d->rab_type != nullptr &&
      cudaMemsetAsync(d_rab_type, 0, sizeof(float) * d->num_types * d->num_types, s) !=
          cudaSuccess)
    return HSTU_ERR_CUDA;
  if (d->num_seqs == 0 || d->total_tokens == 0) return HSTU_OK;
  if (q == nullptr || k == nullptr || v == nullptr || d_o == nullptr || dq == nullptr ||
      dk == nullptr || dv == nullptr)
    return HSTU_ERR_INVALID_ARG;
  if (build_list(ws, w, d->seq_offsets, d->num_seqs, d->total_tokens, d->max_seq_len, d->mask,
                 d->num_candidates, 1, s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  AttnGeom g = make_geom(ws, w, d->timestamps, d->rab_pos, d->max_pos_dist, d->rab_time,
                         d->num_time_buckets, d->num_heads, d->total_tokens, d->mask,
                         d->num_candidates, d->alpha);
  set_types(&g, d->token_types, d->rab_type, d->num_types);
  if (d->rab_type != nullptr) g.d_type = d_rab_type;
  const int grid = max_items(d->total_tokens, d->num_seqs) * d->num_heads;
  // Head width 64 in bf16 with 16-byte aligned rows runs on the tensor cores (bias-gradient bins
  // and table copies in shared memory); every other shape on CUDA cores.
  const bool use_time = d->timestamps != nullptr && d->rab_time != nullptr;
  const bool tc = D == 64 && d->rab_type == nullptr &&
                  attn_uses_tc(D, d->dtype, q, d->ld_q, k, d->ld_k, v, d->ld_v, d_o, d->ld_o) &&
                  aligned16(dq) && aligned16(dk) && aligned16(dv) && (!use_time || aligned16(d->timestamps)) &&
                  attn_bwd_tc_smem(d->rab_pos ? d->max_pos_dist : 0,
                                   d->rab_time ? d->num_time_buckets : 0) <= 227 * 1024;
  cudaError_t e;
  if (tc) {
    CUtensorMap tq, tk, tv, tdo, tts;
    std::memset(&tts, 0, sizeof(tts));
    const int64_t T = d->total_tokens;
    if (!make_map_bf16(&tq, q, T, cols, d->ld_q, 64, kTileRows) ||
        !make_map_bf16(&tk, k, T, cols, d->ld_k, 64, kTileRows) ||
        !make_map_bf16(&tv, v, T, cols, d->ld_v, 64, kTileRows) ||
        !make_map_bf16(&tdo, d_o, T, cols, d->ld_o, 64, kTileRows) ||
        (use_time && !make_map_i64_1d(&tts, d->timestamps, T, attn_bwd_tc_ts_box())))
      return HSTU_ERR_CUDA;
    float* dq_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + w.total_attn);
    CUtensorMap tdq;
    if (!make_map_f32(&tdq, dq_acc, T, cols, cols, 16, 32)) return HSTU_ERR_CUDA;
    const int pgrid = grid < num_sms_current() ? grid : num_sms_current();
    e = launch_attn_bwd_tc(tq, tk, tv, tdo, tts, tdq, g, static_cast<__nv_bfloat16*>(dq), d->ld_q,
                           static_cast<__nv_bfloat16*>(dk), d->ld_k,
                           static_cast<__nv_bfloat16*>(dv), d->ld_v, dq_acc, d_rab_pos,
                           d_rab_time, pgrid, true, zg, s);
    if (zg_applied != nullptr) *zg_applied = zg.q != nullptr;
  } else {
    e = launch_attn_bwd_simt(d->dtype, D, g, q, d->ld_q, k, d->ld_k, v, d->ld_v, d_o, d->ld_o,
                             dq, dk, dv, d_rab_pos, d_rab_time, grid, s);
  }
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}
}  // namespace

extern "C" {

size_t hstu_layer_workspace_size(const hstu_layer_desc_t* d) {
  if (d == nullptr || d->total_tokens < 0 || d->num_seqs < 0 || d->max_seq_len < 0 ||
      d->num_heads < 1 || d->d_qk < 1 || d->d_v < 1)
    return 0;
  const WsLayout w = attn_layout(d->total_tokens, d->num_seqs, d->max_seq_len);
  const size_t es = elem_size(d->dtype);
  const size_t T = static_cast<size_t>(d->total_tokens);
  const size_t n1 = 2 * static_cast<size_t>(d->num_heads) * (d->d_qk + d->d_v);
  const size_t hv = static_cast<size_t>(d->num_heads) * d->d_v;
  return w.total_attn + align_up(T * n1 * es) + 2 * align_up(T * hv * es);
}

}  // extern "C"

namespace {
// One stage of the layer forward (see hstu_layer_forward_stage).  uvqk_ext, when set, takes the
// place of the workspace's f1 output [T, 2H(d_qk+d_v)] (the M-FALCON cache of
// hstu_layer_forward_cached).
hstu_status_t layer_stage(const hstu_layer_desc_t* d, int32_t stage, const void* x,
                          const void* w1, const float* b1, const void* w2, const float* b2,
                          void* y, void* ws, size_t ws_bytes, hstu_stream_t stream,
                          void* uvqk_ext) {
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  if (stage < HSTU_STAGE_F1 || stage > HSTU_STAGE_NORM_GATE_F2) return HSTU_ERR_INVALID_ARG;
  hstu_status_t st = check_common(d->num_seqs, d->total_tokens, d->max_seq_len, d->seq_offsets,
                                  d->num_heads, d->d_qk, d->d_v, d->mask, d->num_candidates,
                                  d->mfalcon_microbatch, d->rab_pos, d->max_pos_dist,
                                  d->rab_time, d->num_time_buckets, d->alpha, d->dtype);
  if (st != HSTU_OK) return st;
  if (d->d_model < 1 || !std::isfinite(d->ln_eps) || d->ln_eps < 0.f) return HSTU_ERR_INVALID_ARG;
  st = check_types(d->token_types, d->rab_type, d->num_types, d->total_tokens);
  if (st != HSTU_OK) return st;
  const int H = d->num_heads, D = d->d_qk, T = d->total_tokens;
  const int hv = H * d->d_v;
  const int n1 = 2 * H * (d->d_qk + d->d_v);
  if (hv > 1024) return HSTU_ERR_UNSUPPORTED;  // LayerNorm row held in one warp's registers
  const size_t need = hstu_layer_workspace_size(d);
  st = check_ws(ws, ws_bytes, need);
  if (st != HSTU_OK) return st;
  if (d->num_seqs == 0 || T == 0) return HSTU_OK;
  if (stage == HSTU_STAGE_F1 && (x == nullptr || w1 == nullptr || !aligned16(x) || !aligned16(w1)))
    return HSTU_ERR_INVALID_ARG;
  if (stage == HSTU_STAGE_NORM_GATE_F2 &&
      (x == nullptr || w2 == nullptr || y == nullptr || x == y || !aligned16(x) ||
       !aligned16(w2) || !aligned16(y)))
    return HSTU_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout w = attn_layout(T, d->num_seqs, d->max_seq_len);
  const size_t es = elem_size(d->dtype);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* uvqk = uvqk_ext != nullptr ? static_cast<uint8_t*>(uvqk_ext) : base + w.total_attn;
  uint8_t* av = base + w.total_attn + align_up(static_cast<size_t>(T) * n1 * es);
  uint8_t* gbuf = av + align_up(static_cast<size_t>(T) * hv * es);
  int32_t* status = reinterpret_cast<int32_t*>(base);
  const uint8_t* u_ptr = uvqk;
  const uint8_t* v_ptr = uvqk + static_cast<size_t>(hv) * es;
  const uint8_t* q_ptr = uvqk + static_cast<size_t>(2 * hv) * es;
  const uint8_t* k_ptr = q_ptr + static_cast<size_t>(H) * d->d_qk * es;

  if (stage == HSTU_STAGE_F1) {
    // f1 + SiLU: [T, d_model] x [d_model, n1] -> uvqk = [U | V | Q | K]
    return gemm(d->dtype, 0, x, d->d_model, w1, n1, T, n1, d->d_model, b1, nullptr, 0, uvqk, n1,
                status, s);
  }
  AttnGeom g = make_geom(ws, w, d->timestamps, d->rab_pos, d->max_pos_dist, d->rab_time,
                         d->num_time_buckets, H, T, d->mask, d->num_candidates, d->alpha);
  set_types(&g, d->token_types, d->rab_type, d->num_types);
  // With the paired attention kernel and the fused output projection, the attention leaves
  // the LayerNorm statistics of each 32-column slice of av in gbuf (decided from the
  // descriptor and the workspace alone, so both stages agree).
  const bool stats_in_attn =
      d->dtype == HSTU_BF16 && hv % 32 == 0 && f2_fused_supported(hv, d->d_model) &&
      aligned16(av) && aligned16(u_ptr) && n1 % 8 == 0 &&
      attn_uses_pair(g, D, attn_uses_tc(D, d->dtype, q_ptr, n1, k_ptr, n1, v_ptr, n1, av, hv));
  if (stage == HSTU_STAGE_ATTENTION) {
    if (stats_in_attn) g.o_stats = reinterpret_cast<float2*>(gbuf);
    return attn_forward_core(ws, w, d->seq_offsets, d->max_seq_len, g, d->num_seqs, T, D,
                             d->dtype, q_ptr, n1, k_ptr, n1, v_ptr, n1, av, hv, s);
  }
  // Norm(AV) ⊙ U, then f2 + residual: Y = X + G W2 + b2
  return norm_gate_f2(d->dtype, av, hv, u_ptr, n1, d->ln_gamma, d->ln_beta, d->ln_eps, w2, b2, x,
                      y, T, hv, d->d_model, gbuf, status, s, stats_in_attn ? hv / 32 : 0);
}
}  // namespace

extern "C" {

hstu_status_t hstu_layer_forward_stage(const hstu_layer_desc_t* d, int32_t stage,
                                       const void* x, const void* w1, const float* b1,
                                       const void* w2, const float* b2, void* y, void* ws,
                                       size_t ws_bytes, hstu_stream_t stream) {
  return layer_stage(d, stage, x, w1, b1, w2, b2, y, ws, ws_bytes, stream, nullptr);
}

hstu_status_t hstu_layer_forward(const hstu_layer_desc_t* d, const void* x, const void* w1,
                                 const float* b1, const void* w2, const float* b2, void* y,
                                 void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  if (x == nullptr || w1 == nullptr || w2 == nullptr || y == nullptr || x == y)
    return d->num_seqs == 0 || d->total_tokens == 0 ? HSTU_OK : HSTU_ERR_INVALID_ARG;
  for (int32_t stage = HSTU_STAGE_F1; stage <= HSTU_STAGE_NORM_GATE_F2; ++stage) {
    const hstu_status_t st =
        hstu_layer_forward_stage(d, stage, x, w1, b1, w2, b2, y, ws, ws_bytes, stream);
    if (st != HSTU_OK) return st;
  }
  return HSTU_OK;
}

size_t hstu_layer_cache_bytes(const hstu_layer_desc_t* d) {
  if (d == nullptr || d->total_tokens < 0 || d->num_heads < 1 || d->d_qk < 1 || d->d_v < 1)
    return 0;
  return static_cast<size_t>(d->total_tokens) * 2 * d->num_heads * (d->d_qk + d->d_v) *
         elem_size(d->dtype);
}

hstu_status_t hstu_layer_forward_cached(const hstu_layer_desc_t* d, const void* x,
                                        const void* w1, const float* b1, const void* w2,
                                        const float* b2, void* y, void* cache, void* ws,
                                        size_t ws_bytes, hstu_stream_t stream) {
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  if (d->num_seqs > 0 && d->total_tokens > 0 && (cache == nullptr || !aligned16(cache)))
    return HSTU_ERR_INVALID_ARG;
  if (x == nullptr || w1 == nullptr || w2 == nullptr || y == nullptr || x == y)
    return d->num_seqs == 0 || d->total_tokens == 0 ? HSTU_OK : HSTU_ERR_INVALID_ARG;
  for (int32_t stage = HSTU_STAGE_F1; stage <= HSTU_STAGE_NORM_GATE_F2; ++stage) {
    const hstu_status_t st =
        layer_stage(d, stage, x, w1, b1, w2, b2, y, ws, ws_bytes, stream, cache);
    if (st != HSTU_OK) return st;
  }
  return HSTU_OK;
}

size_t hstu_layer_candidates_workspace_size(const hstu_layer_desc_t* d) {
  if (d == nullptr || d->total_tokens < 0 || d->num_seqs < 0 || d->max_seq_len < 0 ||
      d->num_heads < 1 || d->d_qk < 1 || d->d_v < 1 || d->num_candidates < 0)
    return 0;
  const WsLayout w = attn_layout(d->total_tokens, d->num_seqs, d->max_seq_len);
  const size_t es = elem_size(d->dtype);
  const size_t bm = static_cast<size_t>(d->num_seqs) * d->num_candidates;
  const size_t n1 = 2 * static_cast<size_t>(d->num_heads) * (d->d_qk + d->d_v);
  const size_t hv = static_cast<size_t>(d->num_heads) * d->d_v;
  // f1 output of the candidates, their row indices, the attention output [T, hv] (the candidate
  // tiles' rows), and the candidates' AV, U and gated norm
  return w.total_attn + align_up(bm * n1 * es) + align_up(bm * 4) +
         align_up(static_cast<size_t>(d->total_tokens) * hv * es) + 3 * align_up(bm * hv * es);
}

hstu_status_t hstu_layer_forward_candidates(const hstu_layer_desc_t* d, const void* x_cand,
                                            const void* w1, const float* b1, const void* w2,
                                            const float* b2, void* y_cand, void* cache,
                                            void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  hstu_status_t st = check_common(d->num_seqs, d->total_tokens, d->max_seq_len, d->seq_offsets,
                                  d->num_heads, d->d_qk, d->d_v, d->mask, d->num_candidates,
                                  d->mfalcon_microbatch, d->rab_pos, d->max_pos_dist,
                                  d->rab_time, d->num_time_buckets, d->alpha, d->dtype);
  if (st != HSTU_OK) return st;
  if (d->mask != HSTU_MASK_MFALCON || d->num_candidates < 1) return HSTU_ERR_INVALID_ARG;
  if (d->d_model < 1 || !std::isfinite(d->ln_eps) || d->ln_eps < 0.f) return HSTU_ERR_INVALID_ARG;
  const int H = d->num_heads, T = d->total_tokens, m = d->num_candidates, B = d->num_seqs;
  const int hv = H * d->d_v, n1 = 2 * H * (d->d_qk + d->d_v), D = d->d_qk;
  if (hv > 1024) return HSTU_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * m > T) return HSTU_ERR_INVALID_ARG;  // every sequence holds m
  st = check_ws(ws, ws_bytes, hstu_layer_candidates_workspace_size(d));
  if (st != HSTU_OK) return st;
  if (B == 0 || T == 0) return HSTU_OK;
  const void* ptrs[] = {x_cand, w1, w2, y_cand, cache};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  if (x_cand == y_cand) return HSTU_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const WsLayout w = attn_layout(T, B, d->max_seq_len);
  const size_t es = elem_size(d->dtype);
  const int bm = B * m;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(base);
  uint8_t* zc = base + w.total_attn;
  int32_t* idx = reinterpret_cast<int32_t*>(zc + align_up(static_cast<size_t>(bm) * n1 * es));
  uint8_t* av = reinterpret_cast<uint8_t*>(idx) + align_up(static_cast<size_t>(bm) * 4);
  uint8_t* avc = av + align_up(static_cast<size_t>(T) * hv * es);
  uint8_t* uc = avc + align_up(static_cast<size_t>(bm) * hv * es);
  uint8_t* gc = uc + align_up(static_cast<size_t>(bm) * hv * es);
  uint8_t* ca = static_cast<uint8_t*>(cache);
  const int nsm = num_sms_current();
  // candidate rows of the jagged layout, then the candidates' f1 output into their cache rows
  cudaError_t e = launch_candidate_rows(d->seq_offsets, B, m, idx, status, s);
  if (e != cudaSuccess) return cuda_fail(e);
  st = gemm(d->dtype, 0, x_cand, d->d_model, w1, n1, bm, n1, d->d_model, b1, nullptr, 0, zc, n1,
            status, s);
  if (st != HSTU_OK) return st;
  e = launch_scatter_rows(zc, static_cast<int64_t>(n1) * es, idx, bm, ca,
                          static_cast<int64_t>(n1) * es, static_cast<int64_t>(n1) * es, nsm, s);
  if (e != cudaSuccess) return cuda_fail(e);
  // attention of the query tiles that hold candidates: the history's K / V come from the cache
  AttnGeom g = make_geom(ws, w, d->timestamps, d->rab_pos, d->max_pos_dist, d->rab_time,
                         d->num_time_buckets, H, T, d->mask, m, d->alpha);
  st = check_types(d->token_types, d->rab_type, d->num_types, T);
  if (st != HSTU_OK) return st;
  set_types(&g, d->token_types, d->rab_type, d->num_types);
  const uint8_t* u_ptr = ca;
  const uint8_t* v_ptr = ca + static_cast<size_t>(hv) * es;
  const uint8_t* q_ptr = ca + static_cast<size_t>(2 * hv) * es;
  const uint8_t* k_ptr = q_ptr + static_cast<size_t>(H) * d->d_qk * es;
  st = attn_forward_core(ws, w, d->seq_offsets, d->max_seq_len, g, B, T, D, d->dtype, q_ptr, n1,
                         k_ptr, n1, v_ptr, n1, av, hv, s, 1);
  if (st != HSTU_OK) return st;
  // the candidates' AV and U rows, Norm(AV) ⊙ U, f2 + residual
  if ((e = launch_gather_rows(av, static_cast<int64_t>(hv) * es, idx, nullptr, bm, avc,
                              static_cast<int64_t>(hv) * es, static_cast<int64_t>(hv) * es, nsm,
                              s)) != cudaSuccess ||
      (e = launch_gather_rows(u_ptr, static_cast<int64_t>(n1) * es, idx, nullptr, bm, uc,
                              static_cast<int64_t>(hv) * es, static_cast<int64_t>(hv) * es, nsm,
                              s)) != cudaSuccess)
    return cuda_fail(e);
  return norm_gate_f2(d->dtype, avc, hv, uc, hv, d->ln_gamma, d->ln_beta, d->ln_eps, w2, b2,
                      x_cand, y_cand, bm, hv, d->d_model, gc, status, s);
}

size_t hstu_layer_backward_workspace_size(const hstu_layer_desc_t* d) {
  if (d == nullptr || d->total_tokens < 0 || d->num_seqs < 0 || d->max_seq_len < 0 ||
      d->num_heads < 1 || d->d_qk < 1 || d->d_v < 1)
    return 0;
  const hstu_attn_desc_t ad = layer_attn_desc(d);
  return layer_bwd_layout(d, ad).total;
}

hstu_status_t hstu_layer_backward(const hstu_layer_desc_t* d, const void* x, const void* w1,
                                  const float* b1, const void* w2, const float* b2,
                                  const void* d_y, void* d_x, float* d_w1, float* d_b1,
                                  float* d_w2, float* d_b2, float* d_rab_pos, float* d_rab_time,
                                  float* d_ln_gamma, float* d_ln_beta, void* ws,
                                  size_t ws_bytes, hstu_stream_t stream) {
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  hstu_status_t st = check_common(d->num_seqs, d->total_tokens, d->max_seq_len, d->seq_offsets,
                                  d->num_heads, d->d_qk, d->d_v, d->mask, d->num_candidates,
                                  d->mfalcon_microbatch, d->rab_pos, d->max_pos_dist,
                                  d->rab_time, d->num_time_buckets, d->alpha, d->dtype);
  if (st != HSTU_OK) return st;
  if (d->d_model < 1 || !std::isfinite(d->ln_eps) || d->ln_eps < 0.f) return HSTU_ERR_INVALID_ARG;
  const int H = d->num_heads, T = d->total_tokens, dm = d->d_model;
  const int hv = H * d->d_v;
  const int n1 = 2 * H * (d->d_qk + d->d_v);
  // tensor-core GEMMs and 16-byte vectors throughout: bf16, widths multiples of 8, LayerNorm
  // rows of 128 .. 1024 features held in one warp
  if (d->dtype != HSTU_BF16 || dm % 8 != 0 || (hv != 128 && hv != 256 && hv != 512 && hv != 1024) ||
      d->rab_type != nullptr)
    return HSTU_ERR_UNSUPPORTED;
  const hstu_attn_desc_t ad = layer_attn_desc(d);
  const LayerBwdLayout L = layer_bwd_layout(d, ad);
  st = check_ws(ws, ws_bytes, L.total);
  if (st != HSTU_OK) return st;
  if ((d->ln_gamma != nullptr && d_ln_gamma == nullptr) ||
      (d->ln_beta != nullptr && d_ln_beta == nullptr) || (b1 != nullptr && d_b1 == nullptr) ||
      (b2 != nullptr && d_b2 == nullptr))
    return HSTU_ERR_INVALID_ARG;
  if (T == 0 || d->num_seqs == 0) return HSTU_OK;
  const void* ptrs[] = {x, w1, w2, d_y, d_x, d_w1, d_w2};
  for (const void* p : ptrs)
    if (p == nullptr || !aligned16(p)) return HSTU_ERR_INVALID_ARG;
  if (x == d_x || d_y == d_x) return HSTU_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* status = reinterpret_cast<int32_t*>(base);
  auto* z = reinterpret_cast<float*>(base + L.z);
  auto* a = reinterpret_cast<__nv_bfloat16*>(base + L.a);
  auto* av = reinterpret_cast<__nv_bfloat16*>(base + L.av);
  auto* g = reinterpret_cast<__nv_bfloat16*>(base + L.g);
  auto* dg = reinterpret_cast<__nv_bfloat16*>(base + L.dg);
  auto* dav = reinterpret_cast<__nv_bfloat16*>(base + L.dav);
  auto* da = reinterpret_cast<__nv_bfloat16*>(base + L.da);
  const size_t attn_ws = L.z;  // the attention calls' part of the workspace
  // column blocks [U | V | Q | K] of the f1 output and of its gradient
  const int64_t offU = 0, offV = hv, offQ = 2 * static_cast<int64_t>(hv),
                offK = offQ + static_cast<int64_t>(H) * d->d_qk;
  const int nsm = num_sms_current();

  // ---- forward, keeping what the backward reads: Z (pre-activation), A = SiLU(Z), AV, G
  st = gemm_tc_layout(3, 0, 1, x, dm, w1, n1, T, n1, dm, 1, b1, nullptr, 0, a, n1, z, n1, nullptr,
                      status, s);
  if (st != HSTU_OK) return st;
  st = hstu_attention_forward(&ad, a + offQ, a + offK, a + offV, av, ws, attn_ws, stream);
  if (st != HSTU_OK) return st;
  if (launch_ln_gate(0, av, hv, a + offU, n1, d->ln_gamma, d->ln_beta, d->ln_eps, g, hv, T, hv,
                     s) != cudaSuccess)
    return HSTU_ERR_CUDA;
  // ---- f2 and the residual edge: dG = dY W2ᵀ, dW2 = Gᵀ dY, db2 = Σ dY
  st = gemm_tc_layout(2, 0, 0, d_y, dm, w2, dm, T, hv, dm, 1, nullptr, nullptr, 0, dg, hv,
                      nullptr, 0, nullptr, status, s);
  if (st != HSTU_OK) return st;
  cudaError_t e = cudaMemsetAsync(d_w2, 0, sizeof(float) * hv * dm, s);
  if (e != cudaSuccess) return cuda_fail(e);
  st = gemm_tc_layout(4, 1, 1, g, hv, d_y, dm, hv, dm, T, weight_grad_splits(hv, dm, T), nullptr,
                      nullptr, 0, nullptr, dm, nullptr, 0, d_w2, status, s);
  if (st != HSTU_OK) return st;
  if (d_b2 != nullptr && (e = launch_colsum(static_cast<const __nv_bfloat16*>(d_y), dm, T, dm,
                                            d_b2, s)) != cudaSuccess)
    return cuda_fail(e);
  // ---- gate and LayerNorm: dU into dA's U block, dAV
  if (d_ln_gamma != nullptr && (e = cudaMemsetAsync(d_ln_gamma, 0, sizeof(float) * hv, s)) != cudaSuccess)
    return cuda_fail(e);
  if (d_ln_beta != nullptr && (e = cudaMemsetAsync(d_ln_beta, 0, sizeof(float) * hv, s)) != cudaSuccess)
    return cuda_fail(e);
  e = launch_ln_gate_bwd(av, hv, a + offU, n1, dg, hv, d->ln_gamma, d->ln_beta, d->ln_eps, dav,
                         hv, da + offU, n1, z + offU, n1, d->ln_gamma ? d_ln_gamma : nullptr,
                         d->ln_beta ? d_ln_beta : nullptr, T, hv, nsm, s);
  if (e != cudaSuccess) return cuda_fail(e);
  // ---- attention: dQ, dK, dV into dA's Q, K, V blocks; the bias-table gradients
  hstu_attn_desc_t bd = ad;
  bd.ld_o = hv;  // dO = dAV
  bool zg_applied = false;
  st = attn_backward_impl(&bd, a + offQ, a + offK, a + offV, dav, da + offQ, da + offK,
                          da + offV, d_rab_pos, d_rab_time, nullptr, ws, attn_ws, stream,
                          SiluGradZ{z + offQ, z + offK, z + offV, n1}, &zg_applied);
  if (st != HSTU_OK) return st;
  // ---- SiLU and f1: dpre = dA ⊙ SiLU'(Z) (already applied to U, and to V, Q, K when the
  // tensor-core backward produced them), dX = dY + dpre W1ᵀ, dW1 = Xᵀ dpre, db1 = Σ dpre
  if (!zg_applied) {
    e = launch_silu_grad_mul(z + offV, n1, da + offV, n1, da + offV, n1, T, n1 - hv, nsm, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  st = gemm_tc_layout(1, 0, 0, da, n1, w1, n1, T, dm, n1, 1, nullptr, d_y, dm, d_x, dm, nullptr,
                      0, nullptr, status, s);
  if (st != HSTU_OK) return st;
  e = cudaMemsetAsync(d_w1, 0, sizeof(float) * dm * n1, s);
  if (e != cudaSuccess) return cuda_fail(e);
  st = gemm_tc_layout(4, 1, 1, x, dm, da, n1, dm, n1, T, weight_grad_splits(dm, n1, T), nullptr,
                      nullptr, 0, nullptr, n1, nullptr, 0, d_w1, status, s);
  if (st != HSTU_OK) return st;
  if (d_b1 != nullptr && (e = launch_colsum(da, n1, T, n1, d_b1, s)) != cudaSuccess)
    return cuda_fail(e);
  (void)b2;  // b2 does not enter any gradient but its own (db2 = Σ dY)
  return HSTU_OK;
}

size_t hstu_stochastic_length_workspace_size(int32_t num_seqs, int32_t total_tokens) {
  if (num_seqs < 0 || total_tokens < 0) return 0;
  return kStatusBytes + align_up(sizeof(int32_t) * static_cast<size_t>(total_tokens)) +
         align_up(sizeof(int32_t) * static_cast<size_t>(num_seqs));
}

hstu_status_t hstu_stochastic_length(const int32_t* seq_offsets, int32_t num_seqs,
                                     int32_t total_tokens, int32_t max_seq_len, int32_t sub_len,
                                     double n_alpha, const float* u, const uint32_t* token_keys,
                                     int32_t* new_offsets, int32_t* kept_index, void* ws,
                                     size_t ws_bytes, hstu_stream_t stream) {
  if (num_seqs < 0 || total_tokens < 0 || max_seq_len < 0 || max_seq_len > kMaxSeqLen ||
      sub_len < 1 || !std::isfinite(n_alpha) || n_alpha < 0.0)
    return HSTU_ERR_INVALID_ARG;
  if (total_tokens > 0 && static_cast<int64_t>(num_seqs) * max_seq_len < total_tokens)
    return HSTU_ERR_INVALID_ARG;
  const hstu_status_t st =
      check_ws(ws, ws_bytes, hstu_stochastic_length_workspace_size(num_seqs, total_tokens));
  if (st != HSTU_OK) return st;
  if (new_offsets == nullptr) return HSTU_ERR_INVALID_ARG;
  if (num_seqs > 0 && (seq_offsets == nullptr || u == nullptr)) return HSTU_ERR_INVALID_ARG;
  if (total_tokens > 0 && (token_keys == nullptr || kept_index == nullptr))
    return HSTU_ERR_INVALID_ARG;
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* local_idx = reinterpret_cast<int32_t*>(base + kStatusBytes);
  int32_t* lens = reinterpret_cast<int32_t*>(
      base + kStatusBytes + align_up(sizeof(int32_t) * static_cast<size_t>(total_tokens)));
  const cudaError_t e = launch_stochastic_length(
      seq_offsets, num_seqs, total_tokens, max_seq_len, sub_len, n_alpha, u, token_keys,
      local_idx, lens, new_offsets, kept_index, reinterpret_cast<int32_t*>(base),
      reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

hstu_status_t hstu_gather_rows(const void* src, int64_t src_row_stride_bytes,
                               const int32_t* index, const int32_t* count, int32_t max_rows,
                               void* dst, int64_t dst_row_stride_bytes, int64_t row_bytes,
                               hstu_stream_t stream) {
  if (max_rows < 0 || row_bytes < 0) return HSTU_ERR_INVALID_ARG;
  if (max_rows == 0 || row_bytes == 0) return HSTU_OK;
  if (src == nullptr || dst == nullptr || index == nullptr) return HSTU_ERR_INVALID_ARG;
  if (row_bytes % 4 != 0 || src_row_stride_bytes % 4 != 0 || dst_row_stride_bytes % 4 != 0 ||
      (reinterpret_cast<uintptr_t>(src) & 3) != 0 || (reinterpret_cast<uintptr_t>(dst) & 3) != 0 ||
      src_row_stride_bytes < row_bytes || dst_row_stride_bytes < row_bytes)
    return HSTU_ERR_INVALID_ARG;
  const cudaError_t e = launch_gather_rows(src, src_row_stride_bytes, index, count, max_rows, dst,
                                           dst_row_stride_bytes, row_bytes, num_sms_current(),
                                           reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

hstu_status_t hstu_jagged_padded_copy(const int32_t* seq_offsets, int32_t num_seqs,
                                      int32_t max_len, const void* jagged,
                                      int64_t jagged_row_stride_bytes, void* padded,
                                      int64_t padded_row_stride_bytes, int64_t row_bytes,
                                      int32_t to_padded, hstu_stream_t stream) {
  if (num_seqs < 0 || max_len < 0 || row_bytes < 0) return HSTU_ERR_INVALID_ARG;
  if (num_seqs == 0 || max_len == 0 || row_bytes == 0) return HSTU_OK;
  if (seq_offsets == nullptr || jagged == nullptr || padded == nullptr) return HSTU_ERR_INVALID_ARG;
  if (row_bytes % 16 != 0 || jagged_row_stride_bytes % 16 != 0 ||
      padded_row_stride_bytes % 16 != 0 || !aligned16(jagged) || !aligned16(padded) ||
      jagged_row_stride_bytes < row_bytes || padded_row_stride_bytes < row_bytes)
    return HSTU_ERR_INVALID_ARG;
  cudaError_t e = launch_jagged_padded(seq_offsets, num_seqs, max_len, jagged,
                                       jagged_row_stride_bytes, padded, padded_row_stride_bytes,
                                       row_bytes, to_padded, num_sms_current(),
                                       reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

hstu_status_t hstu_debug_time_buckets(const int64_t* dt, int32_t n, int32_t* out, int32_t nb,
                                      hstu_stream_t stream) {
  if (n < 0 || nb < 1) return HSTU_ERR_INVALID_ARG;
  if (n == 0) return HSTU_OK;
  if (dt == nullptr || out == nullptr) return HSTU_ERR_INVALID_ARG;
  cudaError_t e = launch_time_buckets(dt, n, out, nb, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

hstu_status_t hstu_debug_bias_index(int32_t rule, const int64_t* in, int32_t n, int32_t param,
                                    int32_t* out, hstu_stream_t stream) {
  if (rule < HSTU_BIAS_RULE_BUCKET64 || rule > HSTU_BIAS_RULE_POS_DIRECT || n < 0)
    return HSTU_ERR_INVALID_ARG;
  const bool time_rule = rule <= HSTU_BIAS_RULE_THRESHOLD;
  if (time_rule ? (param < 1) : (param < 0 || param > kMaxPosDist)) return HSTU_ERR_INVALID_ARG;
  if (n == 0) return HSTU_OK;
  if (in == nullptr || out == nullptr) return HSTU_ERR_INVALID_ARG;
  cudaError_t e =
      launch_bias_index(rule, in, n, param, out, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

hstu_status_t hstu_alibi_tables(float m_p, float m_t, int32_t max_pos_dist,
                                int32_t num_time_buckets, float* rab_pos, float* rab_time) {
  if (!std::isfinite(m_p) || !std::isfinite(m_t) || max_pos_dist < 0 ||
      max_pos_dist > kMaxPosDist || num_time_buckets < 1)
    return HSTU_ERR_INVALID_ARG;
  if (rab_pos != nullptr)
    for (int32_t k = 0; k <= 2 * max_pos_dist; ++k)
      rab_pos[k] = -m_p * static_cast<float>(k - max_pos_dist);
  if (rab_time != nullptr)
    for (int32_t b = 0; b < num_time_buckets; ++b) rab_time[b] = -m_t * static_cast<float>(b);
  return HSTU_OK;
}

hstu_status_t hstu_debug_wait_timeout(void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (check_ws(ws, ws_bytes, kStatusBytes) != HSTU_OK) return HSTU_ERR_WORKSPACE;
  cudaError_t e = launch_wait_timeout_probe(static_cast<int32_t*>(ws),
                                            reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? HSTU_OK : cuda_fail(e);
}

hstu_status_t hstu_workspace_init(void* ws, size_t ws_bytes, hstu_stream_t stream) {
  if (check_ws(ws, ws_bytes, kStatusBytes) != HSTU_OK) return HSTU_ERR_WORKSPACE;
  return cudaMemsetAsync(ws, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
             ? HSTU_OK
             : HSTU_ERR_CUDA;
}

hstu_status_t hstu_sync_status(const void* ws, hstu_stream_t stream) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return HSTU_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int32_t word = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return HSTU_ERR_CUDA;
  if (cudaMemcpy(&word, ws, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (word != 0 && cudaMemset(const_cast<void*>(ws), 0, sizeof(word)) != cudaSuccess)
    return HSTU_ERR_CUDA;
  if (word == 0) return HSTU_OK;
  if (word == HSTU_ERR_TIMEOUT) return HSTU_ERR_TIMEOUT;
  return HSTU_ERR_DEVICE_CHECK;
}

const char* hstu_status_string(hstu_status_t s) {
  switch (s) {
    case HSTU_OK: return "ok";
    case HSTU_ERR_INVALID_ARG: return "invalid argument";
    case HSTU_ERR_UNSUPPORTED: return "unsupported configuration";
    case HSTU_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case HSTU_ERR_CUDA: return "CUDA error";
    case HSTU_ERR_TIMEOUT: return "device wait timed out";
    case HSTU_ERR_DEVICE_CHECK: return "device-side check failed";
  }
  return "unknown status";
}

const char* hstu_version(void) { return "hstu_b200 0.1 sm_100a"; }

const char* hstu_last_error_string(void) { return g_last_error; }

}  // extern "C"

// ---------------------------------------------------------------- built-in scratch variant
// The scratch of hstu_attention_forward_static_ws: a fixed array in every device context that
// loads the library, so that call needs no workspace from its caller.
static __device__ __align__(256) unsigned char g_static_scratch[HSTU_STATIC_SCRATCH_BYTES];

namespace {

constexpr int kMaxScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxScratchDevices] = {};

// Device address of the current device's scratch array, looked up once per device.
hstu_status_t static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxScratchDevices) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "device %d is beyond the %d devices the built-in scratch supports", dev,
                  kMaxScratchDevices);
    return HSTU_ERR_UNSUPPORTED;
  }
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return cuda_fail(e);
    if (p == nullptr || (reinterpret_cast<uintptr_t>(p) % kAlign) != 0) {
      std::snprintf(g_last_error, sizeof(g_last_error),
                    "built-in scratch address is null or not %zu-byte aligned", kAlign);
      return HSTU_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return HSTU_OK;
}

}  // namespace

extern "C" hstu_status_t hstu_attention_forward_static_ws(const hstu_attn_desc_t* d,
                                                          const void* q, const void* k,
                                                          const void* v, void* o,
                                                          int32_t* status_out,
                                                          hstu_stream_t stream) {
  // host-side argument checks first, so a bad call touches no device state
  if (d == nullptr) return HSTU_ERR_INVALID_ARG;
  hstu_status_t st = check_common(d->num_seqs, d->total_tokens, d->max_seq_len, d->seq_offsets,
                                  d->num_heads, d->d_qk, d->d_v, d->mask, d->num_candidates,
                                  d->mfalcon_microbatch, d->rab_pos, d->max_pos_dist,
                                  d->rab_time, d->num_time_buckets, d->alpha, d->dtype);
  if (st != HSTU_OK) return st;
  if (status_out != nullptr && (reinterpret_cast<uintptr_t>(status_out) % 4) != 0)
    return HSTU_ERR_INVALID_ARG;
  // the checks hstu_attention_forward makes before it touches the workspace, made here before
  // the status word of the shared array is cleared
  const int64_t cols = static_cast<int64_t>(d->num_heads) * d->d_qk;
  // (row strides mean nothing for an empty batch: views of zero rows may report any stride)
  if (d->total_tokens > 0 &&
      (d->ld_q < cols || d->ld_k < cols || d->ld_v < cols || d->ld_o < cols))
    return HSTU_ERR_INVALID_ARG;
  if (d->num_seqs > 0 && d->total_tokens > 0 &&
      (q == nullptr || k == nullptr || v == nullptr || o == nullptr))
    return HSTU_ERR_INVALID_ARG;
  const size_t need = hstu_attention_workspace_size(d);
  if (need > HSTU_STATIC_SCRATCH_BYTES) {
    std::snprintf(g_last_error, sizeof(g_last_error),
                  "attention forward needs %zu bytes of scratch, the built-in area holds %zu: "
                  "use hstu_attention_forward with a caller workspace",
                  need, static_cast<size_t>(HSTU_STATIC_SCRATCH_BYTES));
    return HSTU_ERR_WORKSPACE;
  }
  void* ws = nullptr;
  st = static_scratch(&ws);
  if (st != HSTU_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the array keeps the previous call's contents; only the status word must start at zero
  cudaError_t e = cudaMemsetAsync(ws, 0, kStatusBytes, s);
  if (e != cudaSuccess) return cuda_fail(e);
  st = hstu_attention_forward(d, q, k, v, o, ws, HSTU_STATIC_SCRATCH_BYTES, stream);
  if (st != HSTU_OK) return st;
  if (status_out != nullptr) {
    e = cudaMemcpyAsync(status_out, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, s);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return HSTU_OK;
}
