/*
 * hstu.h — C ABI of the B200 (sm_100a) HSTU jagged layer library (libhstu_b200.so).
 *
 * What the library computes (web pages on HSTU, cited by title and section):
 *   [Review §2.1]  "万亿参数推荐大模型：HSTU 架构如何超越传统 Self-Attention", §2.1, the three formulas
 *                  U,V,Q,K = Split(φ1(f1(X)));  A(X)V(X) = φ2(Q Kᵀ + rab_{p,t}) V;
 *                  Y = f2(Norm(A(X)V(X)) ⊙ U(X)), φ1 = φ2 = SiLU, f1/f2 single linear layers,
 *                  and the block diagram's residual edge from the input X to the output Y.
 *   [FunRec 7.1]   "HSTU：Scaling Law 的首次探索", §7.1.4 innovation 1 (pointwise SiLU aggregation,
 *                  no softmax normalisation), innovation 2 (relative bias from position and time
 *                  differences), §7.1.5 M-FALCON (candidates see the whole history but not each
 *                  other; microbatches of b_m candidates; history K/V reused).
 *   [GenRank 6.2]  "6.2 HSTU的工程突破", §6.2.2 (the same candidate mask), §6.2.3 Eq. (6.2.3)
 *                  (relative-bias score; its backward needs the N×N bias gradient).
 *
 * Readings fixed by this library where the pages are silent:
 *   rab_{p,t}(i,j) = rab_pos[clamp(p_i - p_j, -P, P) + P] + rab_time[bucket(t_i - t_j)],
 *   bucket(dt) = clamp(floor(log2(max(1, dt))), 0, NB-1) on int64 (bit-exact), one pair of
 *   tables shared by all heads; score = alpha * <q_i, k_j> + rab (alpha = 1 is the literal
 *   formula); causal mask j <= i; M-FALCON candidates (the last m tokens of each sequence)
 *   all take the position index n = L - m; Norm = LayerNorm over the H*d_v features of a
 *   token, biased variance; split order [U | V | Q | K], head-major within each block.
 *
 * Conventions shared by every entry point:
 *   - Jagged batch: B sequences packed back to back; seq_offsets is int32 [B+1] on the device,
 *     seq_offsets[0] = 0, non-decreasing, seq_offsets[B] = T.  total_tokens (T) and max_seq_len
 *     are host copies, so no call synchronises with the device.  The device re-checks the
 *     offsets; a violation sets the status word (HSTU_ERR_DEVICE_CHECK) and the kernels skip
 *     all work.
 *   - Ownership: the caller allocates and owns every buffer.  The library allocates no device
 *     memory, keeps no global state apart from a per-device cache of driver entry points, and
 *     launches everything on the caller's stream (asynchronous; reentrant per stream).
 *   - Workspace: *_workspace_size() gives the bytes a call needs; ws must be 256-byte aligned.
 *     Its first 256 bytes hold the device status word, which kernels set on a device-side
 *     check failure or a bounded-wait timeout; hstu_sync_status() reports and clears it.
 *     A new workspace is zeroed once with hstu_workspace_init() before its first use.
 *   - Errors: argument errors are found on the host before any launch and returned; a failed
 *     launch returns HSTU_ERR_CUDA.  No entry point aborts the process or traps the GPU.
 *   - Device pointers must be 16-byte aligned and row strides (in elements) such that a row
 *     starts on a 16-byte boundary; otherwise HSTU_ERR_INVALID_ARG.
 *   - Outputs are written, never accumulated into (d_rab_* included).
 */
#ifndef HSTU_B200_H_
#define HSTU_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* hstu_stream_t; /* a cudaStream_t; NULL = the legacy default stream */

typedef enum {
  HSTU_OK = 0,
  HSTU_ERR_INVALID_ARG = 1,   /* a host-side argument check failed; nothing was launched */
  HSTU_ERR_UNSUPPORTED = 2,   /* a valid combination the library does not implement */
  HSTU_ERR_WORKSPACE = 3,     /* ws is NULL, misaligned or smaller than *_workspace_size() */
  HSTU_ERR_CUDA = 4,          /* a CUDA runtime/driver call or a launch failed */
  HSTU_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out (reported via the status word) */
  HSTU_ERR_DEVICE_CHECK = 6   /* a device-side check failed, e.g. malformed seq_offsets */
} hstu_status_t;

typedef enum { HSTU_MASK_CAUSAL = 0, HSTU_MASK_MFALCON = 1 } hstu_mask_t;
typedef enum { HSTU_BF16 = 0, HSTU_FP32 = 1 } hstu_dtype_t;

/* Attention problem over a jagged batch ([Review §2.1] second formula; [FunRec 7.1] §7.1.4-5).
 * Q, K: [T, num_heads * d_qk], V, O: [T, num_heads * d_v], row-major with row strides ld_*
 * (elements), so Q/K/V may be column views of one f1 output.  Head h occupies columns
 * [h*d, (h+1)*d) of its operand. */
typedef struct {
  int32_t num_seqs;           /* B >= 0 */
  int32_t total_tokens;       /* T = seq_offsets[B] (host copy) */
  int32_t max_seq_len;        /* upper bound of every sequence length (host copy) */
  const int32_t* seq_offsets; /* device int32 [B+1] */
  const int64_t* timestamps;  /* device int64 [T] (seconds); NULL disables the time bias */
  int32_t num_heads;          /* H >= 1 */
  int32_t d_qk;               /* per-head query/key width */
  int32_t d_v;                /* per-head value width */
  int64_t ld_q, ld_k, ld_v, ld_o;  /* row strides in elements (not checked when total_tokens is 0) */
  int32_t mask;               /* hstu_mask_t */
  int32_t num_candidates;     /* M-FALCON: the last m tokens of every sequence are candidates */
  int32_t mfalcon_microbatch; /* b_m >= 1 (M-FALCON only); the output does not depend on it */
  const float* rab_pos;       /* device fp32 [2P+1]; NULL disables the position bias */
  int32_t max_pos_dist;       /* P >= 0 */
  const float* rab_time;      /* device fp32 [NB]; NULL disables the time bias */
  int32_t num_time_buckets;   /* NB >= 1 */
  float alpha;                /* scale of <q, k>; 1.0 is the literal formula */
  int32_t dtype;              /* hstu_dtype_t of Q/K/V/O (fp32 accumulation either way) */
  /* Token-type term of bias_{i,j} = f(p_i - p_j, t_i - t_j, type_i, type_j) ("HSTU：Scaling Law
   * 的首次探索" §7.1.4 innovation 2: content and action tokens relate differently), read as a
   * learned table added to the two above: + rab_type[type_i * NT + type_j].  rab_type NULL
   * (the default of a zeroed descriptor) disables it.  Calls with it run the single-tile
   * tensor-core forward (or the CUDA-core kernels) and the CUDA-core backward. */
  const int32_t* token_types; /* device int32 [T], values in [0, NT) */
  const float* rab_type;      /* device fp32 [NT * NT] or NULL */
  int32_t num_types;          /* NT in [1, 64] when rab_type is set */
} hstu_attn_desc_t;

/* Bytes of workspace hstu_attention_forward needs (status word + tile work list). */
size_t hstu_attention_workspace_size(const hstu_attn_desc_t* desc);

/* O_i = Σ_{j visible from i} SiLU(alpha <Q_i, K_j> + rab_{p,t}(i, j)) V_j per head: the
 * pointwise aggregated attention of [Review §2.1] and [FunRec 7.1] §7.1.4 innovation 1, with
 * the causal mask, or the M-FALCON mask of [FunRec 7.1] §7.1.5 / [GenRank 6.2] §6.2.2.
 * q, k, v, o: device pointers of desc->dtype.  Rows of o outside every sequence are not
 * written.  Runs entirely on the stream; no synchronisation. */
hstu_status_t hstu_attention_forward(const hstu_attn_desc_t* desc, const void* q,
                                     const void* k, const void* v, void* o, void* ws,
                                     size_t ws_bytes, hstu_stream_t stream);

/* ---- Built-in scratch variant.  The pages define no such call: it is a library convenience.
 * Size of the scratch area built into the library (one area per device). */
#define HSTU_STATIC_SCRATCH_BYTES ((size_t)1 << 20)

/* hstu_attention_forward without a caller workspace.  For callers that must not allocate device
 * memory once they are running (a serving process whose memory is fully budgeted at start-up,
 * an embedding application with no device allocator of its own, a host thread that may not
 * take an allocator lock): the status word and the tile work list live in a fixed
 * HSTU_STATIC_SCRATCH_BYTES array compiled into the library, so neither the caller nor the
 * library allocates anything.
 *   - Limit: the call needs hstu_attention_workspace_size(desc) bytes; above
 *     HSTU_STATIC_SCRATCH_BYTES (about 65,000 work items: several million tokens) it returns
 *     HSTU_ERR_WORKSPACE before any launch, and hstu_last_error_string() gives both sizes.
 *   - Set-up: the first call on each device looks the array's device address up (with that
 *     device current) and caches it; make that first call before any stream capture begins.
 *     The cached address is never refreshed: after cudaDeviceReset() on a device it is stale,
 *     so do not use this call on that device again in the same process.
 *   - Sharing: every call on a device uses the same array, which keeps the last call's contents;
 *     each call zeroes the status word on its stream first (the work list is rebuilt in full).
 *     Calls that overlap in time on one device (different streams or host threads without
 *     ordering between them) race on the array and give undefined results: order them.
 *   - status_out: optional device int32; when the stream reaches the end of the call it holds
 *     the call's status word (0 when no device-side check fired, HSTU_ERR_TIMEOUT or
 *     HSTU_ERR_DEVICE_CHECK otherwise).  NULL skips the copy.
 * Every other argument and the result are those of hstu_attention_forward. */
hstu_status_t hstu_attention_forward_static_ws(const hstu_attn_desc_t* desc, const void* q,
                                               const void* k, const void* v, void* o,
                                               int32_t* status_out, hstu_stream_t stream);

/* Bytes of workspace hstu_attention_backward needs (adds an fp32 dQ accumulator [T,H,d_qk]). */
size_t hstu_attention_backward_workspace_size(const hstu_attn_desc_t* desc);

/* Gradients of Σ dO ⊙ O through hstu_attention_forward ([GenRank 6.2] §6.2.3: the backward of
 * the N×N relative bias).  With S = alpha QKᵀ + rab and A = SiLU(S) on visible pairs:
 *   dV = Aᵀ dO, dS = (dO Vᵀ) ⊙ SiLU'(S), dQ = alpha dS K, dK = alpha dSᵀ Q,
 *   d_rab_pos[k] = Σ dS over visible pairs with position index k (all heads and sequences),
 *   d_rab_time[b] = Σ dS over visible pairs with time bucket b.
 * d_o uses ld_o; dq/dk/dv use ld_q/ld_k/ld_v.  d_rab_pos / d_rab_time (fp32 [2P+1] / [NB])
 * are overwritten; either may be NULL when the matching table is NULL. */
hstu_status_t hstu_attention_backward(const hstu_attn_desc_t* desc, const void* q,
                                      const void* k, const void* v, const void* d_o, void* dq,
                                      void* dk, void* dv, float* d_rab_pos, float* d_rab_time,
                                      void* ws, size_t ws_bytes, hstu_stream_t stream);

/* hstu_attention_backward with the token-type term: also d_rab_type (fp32 [NT * NT],
 * overwritten) = Σ dS over visible pairs with (type_i, type_j) = (a, b) at a NT + b.  Runs on
 * the CUDA cores.  hstu_attention_backward itself returns HSTU_ERR_INVALID_ARG when
 * desc->rab_type is set (it has no place for that gradient). */
hstu_status_t hstu_attention_backward_typed(const hstu_attn_desc_t* desc, const void* q,
                                            const void* k, const void* v, const void* d_o,
                                            void* dq, void* dk, void* dv, float* d_rab_pos,
                                            float* d_rab_time, float* d_rab_type, void* ws,
                                            size_t ws_bytes, hstu_stream_t stream);

/* One HSTU layer over a jagged batch ([Review §2.1], all three formulas + residual edge). */
typedef struct {
  int32_t num_seqs, total_tokens, max_seq_len;
  const int32_t* seq_offsets;  /* device int32 [B+1] */
  const int64_t* timestamps;   /* device int64 [T]; NULL disables the time bias */
  int32_t d_model;
  int32_t num_heads, d_qk, d_v;
  int32_t mask, num_candidates, mfalcon_microbatch;
  const float* rab_pos;  int32_t max_pos_dist;
  const float* rab_time; int32_t num_time_buckets;
  float alpha;
  float ln_eps;                /* LayerNorm epsilon (1e-5 in every workload here) */
  const float* ln_gamma;       /* fp32 [H*d_v] or NULL (= 1) */
  const float* ln_beta;        /* fp32 [H*d_v] or NULL (= 0) */
  int32_t dtype;               /* hstu_dtype_t of x, w1, w2, y */
  const int32_t* token_types;  /* token-type term, as in hstu_attn_desc_t (NULL rab_type: off) */
  const float* rab_type;
  int32_t num_types;
} hstu_layer_desc_t;

/* Bytes of workspace hstu_layer_forward needs: status + work list + the f1 output
 * [T, 2H(d_qk+d_v)], the attention output [T, H d_v] and the gated norm [T, H d_v]. */
size_t hstu_layer_workspace_size(const hstu_layer_desc_t* desc);

/* Y = X + f2(Norm(A(X)V(X)) ⊙ U(X)) with U,V,Q,K = Split(SiLU(X W1 + b1)) and f2(g) = g W2 + b2.
 * x, y: [T, d_model] row-major (y may not alias x); w1: [d_model, 2H(d_qk+d_v)] row-major;
 * w2: [H d_v, d_model] row-major; b1 / b2: device fp32 [2H(d_qk+d_v)] / [d_model] or NULL.
 * Three kernel stages on the stream: f1 GEMM + SiLU, attention, LayerNorm⊙U, f2 GEMM +
 * residual. */
hstu_status_t hstu_layer_forward(const hstu_layer_desc_t* desc, const void* x, const void* w1,
                                 const float* b1, const void* w2, const float* b2, void* y,
                                 void* ws, size_t ws_bytes, hstu_stream_t stream);

/* ---- M-FALCON cross-request cache ("HSTU：Scaling Law 的首次探索" §7.1.5: the history's K/V are
 * computed once and reused for every later microbatch and request; only candidate rows are new).
 * The cache of one layer is that layer's f1 output [U | V | Q | K] of every token of the jagged
 * batch, [T, 2H(d_qk+d_v)] in desc->dtype, caller-owned (hstu_layer_cache_bytes).
 *   hstu_layer_forward_cached: hstu_layer_forward that keeps its f1 output in cache (prefill).
 *   hstu_layer_forward_candidates: the same layer for the candidates only.  desc describes the
 *     same batch and history as the prefill (same seq_offsets, the M-FALCON mask, m =
 *     num_candidates >= 1 candidates at the end of every sequence, each sequence at least m
 *     long, else the status word reports HSTU_ERR_DEVICE_CHECK); timestamps covers all T tokens
 *     (the candidates' included).  x_cand / y_cand: [B m, d_model], the candidates of sequence 0,
 *     then of sequence 1, ...  The history rows of cache are read, its candidate rows
 *     overwritten; every candidate row of y_cand equals that row of a full
 *     hstu_layer_forward over the history followed by these candidates (history rows never
 *     depend on candidates, so a prefill with other candidates serves as well).  Work: f1 and
 *     f2 on B m rows and the attention of the query tiles that hold candidates.
 * For a stack, each layer has its own cache, and layer l's candidates call takes layer l-1's
 * y_cand as x_cand. */
size_t hstu_layer_cache_bytes(const hstu_layer_desc_t* desc);
hstu_status_t hstu_layer_forward_cached(const hstu_layer_desc_t* desc, const void* x,
                                        const void* w1, const float* b1, const void* w2,
                                        const float* b2, void* y, void* cache, void* ws,
                                        size_t ws_bytes, hstu_stream_t stream);
size_t hstu_layer_candidates_workspace_size(const hstu_layer_desc_t* desc);
hstu_status_t hstu_layer_forward_candidates(const hstu_layer_desc_t* desc, const void* x_cand,
                                            const void* w1, const float* b1, const void* w2,
                                            const float* b2, void* y_cand, void* cache,
                                            void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Bytes of workspace hstu_layer_backward needs: the attention backward's workspace, then the
 * saved forward activations (f1 pre-activation and output [T, 2H(d_qk+d_v)] each, the attention
 * output and the gated norm [T, H d_v] each) and the gradient activations (dG and dAV
 * [T, H d_v], the f1 output's gradient [T, 2H(d_qk+d_v)]). */
size_t hstu_layer_backward_workspace_size(const hstu_layer_desc_t* desc);

/* Gradients of L = Σ d_y ⊙ Y through one layer Y = X + f2(Norm(A(X)V(X)) ⊙ U(X)): the chain rule
 * of [Review §2.1] backwards through f2 and the residual edge, the gate and LayerNorm, the
 * attention ([GenRank 6.2] §6.2.3, the relative-bias gradient), the SiLU and f1 — the training
 * pass over whole user sequences of [FunRec 7.1] §7.1.3.  The forward is recomputed inside the
 * call (nothing is kept between calls), so it needs only the layer's inputs:
 *   d_x = dY + dpre W1ᵀ            bf16 [T, d_model] (may not alias x or d_y)
 *   d_w1 = Xᵀ dpre                 fp32 [d_model, 2H(d_qk+d_v)]
 *   d_b1 = Σ_t dpre                fp32 [2H(d_qk+d_v)]  (required when b1 != NULL, else may be NULL)
 *   d_w2 = Gᵀ dY                   fp32 [H d_v, d_model]
 *   d_b2 = Σ_t dY                  fp32 [d_model]       (may be NULL)
 *   d_rab_pos, d_rab_time          fp32 tables, as hstu_attention_backward (overwritten)
 *   d_ln_gamma, d_ln_beta          fp32 [H d_v], required when ln_gamma / ln_beta are set
 * with dpre = [dU | dV | dQ | dK] ⊙ SiLU'(X W1 + b1).  Every output is overwritten.  bf16 only,
 * no token-type term (HSTU_ERR_UNSUPPORTED when desc->rab_type is set),
 * d_model a multiple of 8 and H d_v in {128, 256, 512, 1024} (else HSTU_ERR_UNSUPPORTED);
 * 16-byte aligned pointers.  Weight gradients are fp32 sums in no fixed order (atomic split-K
 * reduction), so they are reproducible only to rounding. */
hstu_status_t hstu_layer_backward(const hstu_layer_desc_t* desc, const void* x, const void* w1,
                                  const float* b1, const void* w2, const float* b2,
                                  const void* d_y, void* d_x, float* d_w1, float* d_b1,
                                  float* d_w2, float* d_b2, float* d_rab_pos, float* d_rab_time,
                                  float* d_ln_gamma, float* d_ln_beta, void* ws,
                                  size_t ws_bytes, hstu_stream_t stream);

/* Stages of hstu_layer_forward, callable one at a time (e.g. to time each kernel).  The
 * intermediates live in ws at fixed offsets, so the stages must run in order on one workspace:
 *   HSTU_STAGE_F1           uvqk = SiLU(x W1 + b1)                       (tensor-core GEMM)
 *   HSTU_STAGE_ATTENTION    av = attention over the Q/K/V views of uvqk  (work list + kernel)
 *   HSTU_STAGE_NORM_GATE_F2 g = Norm(av) ⊙ U;  y = x + g W2 + b2        (two kernels)
 * Arguments a stage does not read may be NULL. */
typedef enum {
  HSTU_STAGE_F1 = 1,
  HSTU_STAGE_ATTENTION = 2,
  HSTU_STAGE_NORM_GATE_F2 = 3
} hstu_layer_stage_t;

hstu_status_t hstu_layer_forward_stage(const hstu_layer_desc_t* desc, int32_t stage,
                                       const void* x, const void* w1, const float* b1,
                                       const void* w2, const float* b2, void* y, void* ws,
                                       size_t ws_bytes, hstu_stream_t stream);

/* Copy rows between the jagged layout and a padded [B, max_len] layout (row_bytes per row,
 * 16-byte aligned pointers, strides and row_bytes).  to_padded != 0: jagged -> padded, rows
 * past a sequence's end are zero-filled; to_padded == 0: padded -> jagged.  Sequences longer
 * than max_len are truncated (their status is not an error). */
hstu_status_t hstu_jagged_padded_copy(const int32_t* seq_offsets, int32_t num_seqs,
                                      int32_t max_len, const void* jagged,
                                      int64_t jagged_row_stride_bytes, void* padded,
                                      int64_t padded_row_stride_bytes, int64_t row_bytes,
                                      int32_t to_padded, hstu_stream_t stream);

/* Stochastic Length of "HSTU：Scaling Law 的首次探索" §7.1.5: long sequences are, at random,
 * replaced by a shorter subsequence while training, which cuts the attention's O(n²) work.  The
 * page's formula is garbled; this library reads it as: a sequence of n tokens stays whole when
 * n <= N^{α/2}; otherwise, with probability 1 - N^α / n², it is replaced by sub_len =
 * floor(N^{α/2}) of its tokens in their original order, else it stays whole (N the longest length
 * the data allows, α in (1, 2]; α = 2 never truncates).  The page picks the subsequence "by
 * feature weighting" without saying how; here it is uniformly random: the sub_len tokens with
 * the smallest token_keys (ties to the lower index).
 *   sub_len = floor(N^{α/2}) >= 1 and n_alpha = N^α are computed by the caller, so that the
 *   decision u[b] < 1 - n_alpha / n² is the same fp64 expression everywhere.
 *   u: device fp32 [B], uniform draws on [0, 1), one per sequence; token_keys: device uint32 [T],
 *   random keys (the random numbers are inputs: the result is a pure function of them).
 *   new_offsets: device int32 [B+1] out, the offsets of the kept tokens; kept_index: device
 *   int32 [T] out, the global indices of the kept tokens in the new order (its first
 *   new_offsets[B] entries are written).  ws: hstu_stochastic_length_workspace_size bytes
 *   (status word first; zero it once with hstu_workspace_init).  Malformed seq_offsets set the
 *   status word (HSTU_ERR_DEVICE_CHECK) and those sequences keep no token.
 * New total and lengths live on the device; read new_offsets back when the host needs them.
 * hstu_gather_rows then moves any per-token array (embeddings, timestamps) to the new layout. */
size_t hstu_stochastic_length_workspace_size(int32_t num_seqs, int32_t total_tokens);
hstu_status_t hstu_stochastic_length(const int32_t* seq_offsets, int32_t num_seqs,
                                     int32_t total_tokens, int32_t max_seq_len, int32_t sub_len,
                                     double n_alpha, const float* u, const uint32_t* token_keys,
                                     int32_t* new_offsets, int32_t* kept_index, void* ws,
                                     size_t ws_bytes, hstu_stream_t stream);

/* dst row r = src row index[r] for r < min(*count, max_rows) (count: device int32, e.g.
 * &new_offsets[B] of hstu_stochastic_length; NULL gathers max_rows rows).  index: device int32.
 * Rows of row_bytes bytes; pointers, strides and row_bytes multiples of 4 (16-byte vectors when
 * all are multiples of 16).  Asynchronous on stream. */
hstu_status_t hstu_gather_rows(const void* src, int64_t src_row_stride_bytes,
                               const int32_t* index, const int32_t* count, int32_t max_rows,
                               void* dst, int64_t dst_row_stride_bytes, int64_t row_bytes,
                               hstu_stream_t stream);

/* Tables for the parameter-free relative bias of "6.2 HSTU的工程突破" §6.2.3, Eq. (6.2.6):
 * bias(i, j) = -m_p (p_i - p_j) - m_t bucket(t_i - t_j).  The bias is linear in the integer
 * position difference and in the bucket index, so it is the learned-table bias with
 * rab_pos[k] = -m_p (k - P) (k = 0 .. 2P) and rab_time[b] = -m_t b (b = 0 .. NB-1): pass these
 * tables to the attention or layer calls with max_pos_dist = P.  The position term is exact only
 * where |p_i - p_j| <= P, so take P >= the longest sequence length - 1.  Host arrays owned by the
 * caller, [2P+1] and [NB] floats; either may be NULL to skip it.  Returns HSTU_ERR_INVALID_ARG
 * for a non-finite slope, P < 0, P > 2^24 or NB < 1; no device work.
 * Speed note: the paired head-width-64 forward keeps a 4-wide copy of the position table in
 * shared memory, which fits for P up to about 1100; a larger P (these tables with sequences
 * longer than that) runs the single-tile tensor-core forward, which reads the table from global
 * memory and is slower but computes the same result. */
hstu_status_t hstu_alibi_tables(float m_p, float m_t, int32_t max_pos_dist,
                                int32_t num_time_buckets, float* rab_pos, float* rab_time);

/* Failure-path check of the status word: launches one CTA that waits, with the bounded wait
 * every kernel of the library uses, on a barrier phase that nothing completes.  The wait gives
 * up after its limit (2 s), writes HSTU_ERR_TIMEOUT into the status word of ws and the kernel
 * returns; the next hstu_sync_status(ws) reports HSTU_ERR_TIMEOUT and clears the word, and the
 * context stays usable.  ws: device workspace of at least 256 bytes, 256-byte aligned, owned by
 * the caller.  Returns HSTU_ERR_WORKSPACE for a missing, misaligned or short ws (nothing is
 * launched), HSTU_ERR_CUDA if the launch fails, else HSTU_OK (asynchronous on stream). */
hstu_status_t hstu_debug_wait_timeout(void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Debug export of the time-bias bucket rule: out[i] = clamp(floor(log2(max(1, dt[i]))), 0,
 * nb-1), computed on the device by the same code the attention kernels inline, so it can be
 * compared bit-exactly with an integer reference.  dt, out: device [n]. */
hstu_status_t hstu_debug_time_buckets(const int64_t* dt, int32_t n, int32_t* out, int32_t nb,
                                      hstu_stream_t stream);

/* Debug export of every integer rule the attention kernels use to turn a (query, key) pair into
 * bias-table indices ("HSTU：Scaling Law 的首次探索" §7.1.4 innovation 2: a bias from the position
 * and time differences).  The kernels fold these indices into their epilogues in several forms;
 * this call evaluates each form with the very device functions the kernels call, so that a test
 * can compare them bit for bit with an integer reference:
 *   rule HSTU_BIAS_RULE_BUCKET64    in[i] = dt (any int64), param = NB: the 64-bit bucket
 *                                   clamp(floor(log2(max(1, dt))), 0, NB-1) (M-FALCON segments,
 *                                   the backward, the single-tile forward).
 *   rule HSTU_BIAS_RULE_BUCKET_ROW  in[i] = dt with |dt| < 2^23, param = NB: the per-row bucket
 *                                   bounds of the paired forward (fp32-exponent method).
 *   rule HSTU_BIAS_RULE_TIME_ELEM   in[i] = dt with |dt| < 2^23, param = NB: the time-table entry
 *                                   the paired forward's per-element path reads (its 64-entry
 *                                   table repeats bucket NB-1 past the end).
 *   rule HSTU_BIAS_RULE_BUCKET_CLS  in[i] = dt with |dt| < 2^31, param = NB: the paired forward's
 *                                   tile classifier (count of leading zeros on 32 bits).
 *   rule HSTU_BIAS_RULE_THRESHOLD   in[3i..3i+2] = (dt_lo, dt_hi, dt), dt_lo <= dt <= dt_hi, all
 *                                   within +-2^23, param = NB: the bucket the two-bucket path
 *                                   picks for dt in a row whose keys span [dt_lo, dt_hi]; -1 when
 *                                   the row spans more than two buckets (the kernel then takes
 *                                   the per-element path).
 *   rule HSTU_BIAS_RULE_POS_TABLE   in[3i..] = (p_i, j, unused), param = P: the rab_pos index the
 *                                   paired forward reads for query position p_i and key j through
 *                                   its 4-wide shifted table (tile of 96 keys, lane j mod 4).
 *   rule HSTU_BIAS_RULE_POS_GENERAL in[3i..] = (p_i, j, n), param = P: the index of the M-FALCON
 *                                   candidate segments (key position min(j, n)).
 *   rule HSTU_BIAS_RULE_POS_SEGMENT in[3i..] = (p_min, j_last, unused), param = P: 2P when the
 *                                   classifier gives a row segment (smallest query position
 *                                   p_min, last key j_last) one constant position term, else -1.
 *   rule HSTU_BIAS_RULE_POS_DIRECT  in[3i..] = (p_i, p_j, unused), param = P: clamp(p_i - p_j,
 *                                   -P, P) + P as the backward and CUDA-core kernels form it.
 * in: device int64 [n] (rules 0-3) or [3n] (rules 4-8); out: device int32 [n].  Returns
 * HSTU_ERR_INVALID_ARG for an unknown rule, n < 0, NB < 1 or P outside [0, 2^24]. */
typedef enum {
  HSTU_BIAS_RULE_BUCKET64 = 0,
  HSTU_BIAS_RULE_BUCKET_ROW = 1,
  HSTU_BIAS_RULE_TIME_ELEM = 2,
  HSTU_BIAS_RULE_BUCKET_CLS = 3,
  HSTU_BIAS_RULE_THRESHOLD = 4,
  HSTU_BIAS_RULE_POS_TABLE = 5,
  HSTU_BIAS_RULE_POS_GENERAL = 6,
  HSTU_BIAS_RULE_POS_SEGMENT = 7,
  HSTU_BIAS_RULE_POS_DIRECT = 8
} hstu_bias_rule_t;

hstu_status_t hstu_debug_bias_index(int32_t rule, const int64_t* in, int32_t n, int32_t param,
                                    int32_t* out, hstu_stream_t stream);

/* Zero the status word at the start of ws (asynchronously, on the stream).  Call once on a new
 * workspace before its first use: the status word must start at zero. */
hstu_status_t hstu_workspace_init(void* ws, size_t ws_bytes, hstu_stream_t stream);

/* Synchronise the stream, read the status word kept in ws (a workspace previously passed to
 * a compute call), clear it, and return it (HSTU_OK if no device-side check fired). */
hstu_status_t hstu_sync_status(const void* ws, hstu_stream_t stream);

/* Text of the last CUDA error this library saw on the calling thread ("" if none); useful
 * after HSTU_ERR_CUDA.  The string stays valid until the thread's next library call. */
const char* hstu_last_error_string(void);

/* Human-readable name of a status code (static string). */
const char* hstu_status_string(hstu_status_t status);

/* Library version string, e.g. "hstu_b200 0.1 sm_100a". */
const char* hstu_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HSTU_B200_H_ */
