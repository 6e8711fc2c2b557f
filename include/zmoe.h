/*
 * libzmoe: the sparse mixture-of-experts feed-forward path of the ZONOS2
 * autoregressive decoder, as hand-written CUDA kernels for NVIDIA B200 (sm_100a).
 *
 * Sources (the ZONOS2 pages):
 *   [DIGEST]  "ZONOS2 Technical Report" digest (audio-paper-digest blog),
 *             section "method overview and architecture": item 1 (delay pattern over
 *             N = 9 DAC codebooks), item 5 (input = RMSNorm of the summed codebook
 *             embeddings; 28 layers, MoE layers with 16 experts, top-1 routing,
 *             top-2 in the last MoE layer), item 6 (per-layer bias b_l that steers
 *             expert usage toward uniform).
 *   [ABSTRACT] "ZONOS2 Technical Report" (mlsanity.com), Abstract (8B total, 900M
 *             active) and "Builds on" (GLU Variants Improve Transformer; Root Mean
 *             Square Layer Normalization; Auxiliary-Loss-Free Load Balancing).
 *   [ROUTING] telknet.cc article on ZONOS2, section 2.1 (routing intuition: linear
 *             router, SiLU, TopK; the printed equation was lost in extraction).
 *
 * Conventions for every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  No call
 *     allocates or frees device memory; scratch comes from caller-provided
 *     `workspace` / `ws_bytes`, sized by the matching *_workspace_size() query.
 *   - Every call is asynchronous on `stream` (NULL = the legacy default stream) and
 *     never synchronises.  Results are valid once the stream reaches the call.
 *   - Row-major layouts throughout.  Activations [T, d]; router W_r [E, d];
 *     W_gate, W_up [E, f, d] and W_down [E, d, f] (every weight row is contiguous
 *     along the contraction dimension, i.e. K-major).
 *   - Arguments are checked on the host before anything is launched; a bad argument
 *     returns ZMOE_ERR_INVALID_ARG (or ZMOE_ERR_UNSUPPORTED for a valid but unbuilt
 *     shape) and launches nothing.  A launch failure returns ZMOE_ERR_CUDA;
 *     zmoe_last_error() then gives the CUDA message (thread-local).
 *   - Data errors found on the device (an id or expert index out of range) never
 *     fault: the offending element is skipped and a device error counter is
 *     incremented; read it with zmoe_get_device_errors().
 *   - Sizes are int; T * max(d, f) and T * k must fit in int32.
 */
#ifndef ZMOE_H
#define ZMOE_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZMOE_API __attribute__((visibility("default")))
#else
#define ZMOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* zmoe_stream_t;

typedef enum {
  ZMOE_OK = 0,
  ZMOE_ERR_INVALID_ARG = 1,        /* checked on the host, nothing launched          */
  ZMOE_ERR_UNSUPPORTED = 2,        /* valid arguments, shape or dtype not built      */
  ZMOE_ERR_CUDA = 3,               /* CUDA runtime error; see zmoe_last_error()      */
  ZMOE_ERR_WORKSPACE_TOO_SMALL = 4,
  ZMOE_ERR_DEVICE_CHECK = 5,       /* device-side data check failed (counter > 0)    */
  ZMOE_ERR_TIMEOUT = 6             /* a bounded device-side wait gave up             */
} zmoe_status;

typedef enum {
  ZMOE_F32 = 0,
  ZMOE_BF16 = 1
} zmoe_dtype;

/* Library version, as 10000 * major + 100 * minor + patch. */
ZMOE_API int zmoe_version(void);

/* Static text for a status code. */
ZMOE_API const char* zmoe_status_string(int status);

/* Message of the last failing call on this host thread ("" when none). */
ZMOE_API const char* zmoe_last_error(void);

/*
 * Delay pattern, [DIGEST] item 1:  Y[b, t, j] = X[b, t - j, j]  when 0 <= t - j < T,
 * and `pad` elsewhere.
 *   X: int32 [B, T, N]  ->  Y: int32 [B, T + N - 1, N].
 * B >= 0, T >= 0, 1 <= N <= 64.  Every id is copied bit-exactly.
 */
ZMOE_API zmoe_status zmoe_delay_shear(const int32_t* X, int32_t* Y, int B, int T, int N, int32_t pad,
                             zmoe_stream_t stream);

/*
 * Inverse delay pattern, [DIGEST] item 1:  X_hat[b, t, j] = Y[b, t + j, j].
 *   Y: int32 [B, Ty, N]  ->  X_hat: int32 [B, Ty - N + 1, N].   Requires Ty >= N - 1.
 */
ZMOE_API zmoe_status zmoe_delay_unshear(const int32_t* Y, int32_t* X, int B, int Ty, int N, zmoe_stream_t stream);

/*
 * Summed codebook embeddings followed by RMSNorm, [DIGEST] item 5 (RMSNorm as in
 * "Root Mean Square Layer Normalization", [ABSTRACT] "Builds on"):
 *   e[t] = sum_{j < N} tables[j, ids[t, j], :]              (fp32 sum)
 *   out[t] = e[t] / sqrt(mean_c e[t, c]^2 + eps) * gamma
 *   ids: int32 [T, N], each in [0, V) (V = 1025: ids 0..1023 plus the pad id 1024);
 *   tables: [N, V, d] of `table_dtype`; gamma: f32 [d]; out: [T, d] of `out_dtype`.
 *   d % 8 == 0.  An id outside [0, V) contributes nothing and counts a device error.
 *   tables, out: 16-byte aligned.
 */
ZMOE_API zmoe_status zmoe_embed_sum_rmsnorm(const int32_t* ids, const void* tables, zmoe_dtype table_dtype,
                                   const float* gamma, float eps, int T, int N, int V, int d,
                                   void* out, zmoe_dtype out_dtype, zmoe_stream_t stream);

/*
 * RMSNorm of each row (the per-layer pre-norm of the decode stack):
 *   out[t] = h[t] / sqrt(mean_c h[t, c]^2 + eps) * gamma
 *   h: [T, d] of `in_dtype`; gamma: f32 [d]; out: [T, d] of `out_dtype`.  d % 8 == 0,
 *   16-byte aligned h and out.
 */
ZMOE_API zmoe_status zmoe_rmsnorm(const void* h, zmoe_dtype in_dtype, const float* gamma, float eps, int T, int d,
                         void* out, zmoe_dtype out_dtype, zmoe_stream_t stream);

/*
 * Router with a selection-only bias, [DIGEST] items 5-6, [ROUTING] section 2.1,
 * [ABSTRACT] "Builds on" (Auxiliary-Loss-Free Load Balancing):
 *   l = W_r x (fp32 accumulation);  q = l + logit_bias;  s = q + sel_bias;
 *   expert_idx[t, :] = the k largest s, by descending s, ties -> lower expert index;
 *   p = softmax(q) over all E;  k == 1: gates = p[sel];
 *   k == 2: gates_i = p[sel_i] / (p[sel_0] + p[sel_1]).
 *   margin[t] (optional) = s_(1) - s_(2) for k == 1, min(s_(1) - s_(2), s_(2) - s_(3))
 *   for k == 2 (+inf when E == k).
 *   x: [T, d], w_router: [E, d], both of `dtype`; logit_bias, sel_bias: f32 [E] or NULL
 *   (= zeros); expert_idx: int32 [T, k]; gates: f32 [T, k]; margin: f32 [T] or NULL.
 *   1 <= E <= 64, k in {1, 2}, k <= E, d % 8 == 0; x and w_router 16-byte aligned.
 *   w_router (and x) may be NULL when E == 1 (a dense FFN layer): every token then gets expert 0
 *   with gate 1 and margin +inf.
 */
ZMOE_API zmoe_status zmoe_route(const void* x, const void* w_router, zmoe_dtype dtype, const float* logit_bias,
                       const float* sel_bias, int T, int d, int E, int k, int32_t* expert_idx, float* gates,
                       float* margin, zmoe_stream_t stream);

/* Bytes of workspace zmoe_permute needs for these sizes. */
ZMOE_API size_t zmoe_permute_workspace_size(int T, int E, int k);

/*
 * Dispatch permutation (implied by sparse experts, [DIGEST] item 5):
 *   counts[e]  = #{(t, i) : expert_idx[t, i] == e}            int32 [E]
 *   offsets    = exclusive prefix sum of counts                int32 [E + 1]
 *   rows ordered by expert, then by token (stable, deterministic):
 *   perm[row] = t                                              int32 [T * k]
 *   inv_perm[t, i] = row holding assignment (t, i)             int32 [T, k]
 *   x_perm[row] = x[perm[row]]                                 [T * k, d] of `dtype`
 * Bit-exact and deterministic.  An expert index outside [0, E) counts a device error;
 * that assignment is dropped (its inv_perm entry is -1) and the rows after it in the
 * same expert are unaffected.  d % 8 == 0; x, x_perm 16-byte aligned.
 */
ZMOE_API zmoe_status zmoe_permute(const int32_t* expert_idx, const void* x, zmoe_dtype dtype, int T, int d, int E, int k,
                         int32_t* counts, int32_t* offsets, int32_t* perm, int32_t* inv_perm, void* x_perm,
                         void* workspace, size_t ws_bytes, zmoe_stream_t stream);

/*
 * zmoe_permute without any device allocation, for callers that cannot allocate: code whose
 * device memory is wholly owned by a host framework's pool allocator (a cudaMalloc behind the
 * pool's back can fail for lack of memory, or stall every stream while the driver maps the
 * pages), and code on a latency-critical path that must never synchronise the device.  The
 * ZONOS2 pages have no counterpart: this is an interface convenience, not a step of the method.
 *   Same arguments, outputs and results as zmoe_permute, without workspace/ws_bytes.
 *   Its scratch (per-tile expert counts, 64 KB) is a static device array inside the
 *   library, held by every GPU that loads it until the process exits.  Limit: T * k <=
 *   65536; larger problems return ZMOE_ERR_INVALID_ARG with a message naming the limit and
 *   launch nothing.  The first call on a device looks up that array's device address (once
 *   per device, with the device current) and caches it for the life of the process, so a
 *   device reset after that first call is not supported; make the first call before any
 *   stream capture.  All calls share the array and it keeps the last call's contents (the
 *   call rewrites every entry it reads, so nothing needs clearing between calls); calls that
 *   overlap on the GPU (different streams without ordering between them) race on it and give
 *   wrong results.  It calls no cudaMalloc, cudaFree or allocating library routine.
 */
ZMOE_API zmoe_status zmoe_permute_noalloc(const int32_t* expert_idx, const void* x, zmoe_dtype dtype, int T, int d,
                                          int E, int k, int32_t* counts, int32_t* offsets, int32_t* perm,
                                          int32_t* inv_perm, void* x_perm, zmoe_stream_t stream);

/*
 * One-time preparation of the down-projection weights for the f16 prefill path (no counterpart on
 * the pages: a storage format of the weights).  Both operands of a tensor-core MMA share one 16-bit
 * format, and the prefill down GEMM carries h in f16 (11 significant bits; one bf16 h costs up to 3%
 * of the output RMS), so W_down is converted once to f16, each expert scaled by a power of two that
 * puts its largest |w| in [2^14, 2^15):
 *   w_down_f16[e] = f16(w_down[e] * 2^s_e),   down_scale[e] = 2^-s_e
 * exact for every weight within 2^28 of the expert's largest (smaller ones round with an absolute
 * error below 2^-39 of the largest).  w_down: bf16 [E, d, f]; w_down_f16: f16 [E, d, f] (caller
 * memory, 16-byte aligned); down_scale: f32 [E]; workspace: >= 4 E bytes of device scratch.
 */
ZMOE_API zmoe_status zmoe_prepare_w_down_f16(const void* w_down, int E, int d, int f, void* w_down_f16,
                                             float* down_scale, void* workspace, size_t ws_bytes,
                                             zmoe_stream_t stream);

/*
 * The grouped SwiGLU of zmoe_grouped_swiglu for prefill-size batches with h carried in f16 and the
 * prepared down weights (zmoe_prepare_w_down_f16):
 *   h[r]      = f16(silu(W_gate[e] x_perm[r]) * (W_up[e] x_perm[r]))             [f] f16
 *   y_perm[r] = down_scale[e] * (W_down_f16[e] h[r])                              [d] f32
 * x_perm, w_gate, w_up: bf16 as zmoe_grouped_swiglu; w_down_f16: f16 [E, d, f]; down_scale: f32 [E];
 * h: f16 [M_total, f] (caller scratch that also exposes the hidden activations); offsets on the device.
 * An |h| beyond f16's range (65504) counts a device error (zmoe_get_device_errors).  Runs the CTA-pair
 * tcgen05 kernels at any M_total (built for >= 64 rows per expert on average); d % 256 == 0,
 * f % 256 == 0, 16-byte aligned.  No workspace.
 */
ZMOE_API zmoe_status zmoe_grouped_swiglu_f16h(const void* x_perm, const int32_t* offsets, int M_total,
                                              const void* w_gate, const void* w_up, const void* w_down_f16,
                                              const float* down_scale, int E, int d, int f, void* h, float* y_perm,
                                              zmoe_stream_t stream);

/* Bytes of workspace zmoe_grouped_swiglu needs for these sizes. */
ZMOE_API size_t zmoe_grouped_swiglu_workspace_size(int M_total, int E, int d, int f, zmoe_dtype dtype);

/*
 * Per-expert SwiGLU over the permuted rows ("GLU Variants Improve Transformer",
 * [ABSTRACT] "Builds on"; SiLU per [ROUTING] section 2.1):
 *   for each expert e and each row r in [offsets[e], offsets[e + 1]):
 *     h[r]      = silu(W_gate[e] x_perm[r]) * (W_up[e] x_perm[r])     [f]
 *     y_perm[r] = W_down[e] h[r]                                      [d], stored as f32
 *   silu(z) = z / (1 + exp(-z)); contractions accumulate in fp32.
 *   bf16: h is kept as a pair of bf16 values, h_hi = bf16(h) and h_lo = bf16(h - h_hi),
 *   stored side by side as h: bf16 [M_total, 2 f] (columns [0, f) = h_hi, [f, 2 f) = h_lo),
 *   and y_perm = W_down h_hi + W_down h_lo: both tensor-core operands stay bf16 while h
 *   carries ~16 significant bits into the second contraction.
 *   f32: h is f32 [M_total, f].
 *   x_perm: [M_total, d]; offsets: int32 [E + 1] on the DEVICE (read by the kernels,
 *   never copied to the host); M_total = T * k is the host-side row bound and must be
 *   >= offsets[E]; w_gate, w_up: [E, f, d]; w_down: [E, d, f]; h: caller scratch (above)
 *   that also exposes the hidden activations; y_perm: f32 [M_total, d].  Rows at or past
 *   offsets[E] are neither read into results nor written.
 *   bf16: d % 256 == 0, f % 256 == 0; f32: d % 4 == 0, f % 4 == 0.  16-byte aligned.
 */
ZMOE_API zmoe_status zmoe_grouped_swiglu(const void* x_perm, const int32_t* offsets, int M_total, const void* w_gate,
                                const void* w_up, const void* w_down, zmoe_dtype dtype, int E, int d, int f,
                                void* h, float* y_perm, void* workspace, size_t ws_bytes, zmoe_stream_t stream);

/*
 * Gate-weighted combine ([ROUTING] section 2.1: the output is the gate-weighted sum of
 * the chosen experts), as a per-token gather in fixed slot order (deterministic):
 *   y[t] = residual[t] + sum_{i < k} gates[t, i] * y_perm[inv_perm[t, i]]
 *   y_perm: f32 [T * k, d]; inv_perm: int32 [T, k]; gates: f32 [T, k];
 *   residual: f32 [T, d] or NULL (= zeros); y: f32 [T, d] (may alias residual).
 *   An inv_perm entry outside [0, T * k) contributes nothing and counts a device error.
 *   d % 4 == 0, 16-byte aligned y_perm, residual, y.
 */
ZMOE_API zmoe_status zmoe_combine(const float* y_perm, const int32_t* inv_perm, const float* gates, const float* residual,
                         int T, int d, int k, float* y, zmoe_stream_t stream);

/* Bytes of workspace zmoe_moe_layer needs for these sizes (0 for T == 0 or bad arguments). */
ZMOE_API size_t zmoe_moe_layer_workspace_size(int T, int d, int f, int E, int k, zmoe_dtype dtype);

/*
 * One sparse MoE layer, optionally with its pre-norm ([DIGEST] items 5-6: RMSNorm, sparse
 * MoE FFN with top-1 routing and top-2 in the last layer; [ROUTING] section 2.1: router,
 * gate-weighted sum of the chosen experts' SwiGLU outputs):
 *   gamma != NULL:  x = RMSNorm(h) * gamma = h / sqrt(mean_c h^2 + eps) * gamma, rounded to
 *                   `dtype` (the decode stack's pre-norm residual block); `x` is not read.
 *   gamma == NULL:  x is the layer input.
 *   y[t] = h[t] + sum_{i < k} gates[t, i] * FFN_{expert_idx[t, i]}(x[t])   (h == NULL: no residual)
 * with the router, dispatch, SwiGLU and combine of zmoe_route, zmoe_permute,
 * zmoe_grouped_swiglu and zmoe_combine (same conventions, same results up to fp32 summation
 * order).  A few tokens (bf16, T * k <= 4) run as one cooperative launch that contracts every
 * weight row whole on one SM (the hidden activations kept in fp32, not as a bf16 pair); decode
 * sizes (bf16, T * k < 64 E, T * k <= 1024, d and f multiples of 256) run as one cooperative
 * stream-K launch; other sizes run those entry points in order.
 *   x: [T, d] of `dtype` (or NULL with gamma); h: f32 [T, d] or NULL (required with gamma);
 *   gamma: f32 [d] or NULL; w_router [E, d], w_gate, w_up [E, f, d], w_down [E, d, f] of
 *   `dtype`; logit_bias, sel_bias: f32 [E] or NULL.
 *   Outputs: y: f32 [T, d] (may alias h); expert_idx int32 [T, k], gates f32 [T, k],
 *   margin f32 [T] (as zmoe_route) and x_norm [T, d] of `dtype` (the routed input, with
 *   gamma only) are optional (NULL: kept in the workspace).
 *   w_router may be NULL when E == 1: the layer is then the dense SwiGLU FFN of the decoder's
 *   dense layers (gate 1), [DIGEST] item 5 (layers 0-2 and 27 are dense).
 *   workspace: zmoe_moe_layer_workspace_size() bytes, 256-byte aligned; it also holds the
 *   intermediates (x_perm, the hidden activations, y_perm).  1 <= E <= 64, k in {1, 2},
 *   k <= E, d % 8 == 0, f % 8 == 0 (bf16: multiples of 256); 16-byte aligned pointers.
 */
ZMOE_API zmoe_status zmoe_moe_layer(const void* x, const float* h, const float* gamma, float eps,
                                    const void* w_router, const float* logit_bias, const float* sel_bias,
                                    const void* w_gate, const void* w_up, const void* w_down, zmoe_dtype dtype,
                                    int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                                    float* gates, float* margin, void* x_norm, void* workspace, size_t ws_bytes,
                                    zmoe_stream_t stream);

/* Bytes of workspace zmoe_moe_layer_fp8 needs (0 when the sizes are not decode sizes). */
ZMOE_API size_t zmoe_moe_layer_fp8_workspace_size(int T, int d, int f, int E, int k);

/*
 * zmoe_moe_layer with fp8 expert weights (the pages' serving stack runs the model in fp8: ZONOS2
 * page of the sglang-omni cookbook, "Benchmark Results"): each expert weight row is stored as E4M3
 * codes (bias 7, no infinities) with one fp32 scale, w = code * scale.  The router stays in bf16.
 *   q_gate, q_up: uint8 [E, f, d]; q_down: uint8 [E, d, f]; s_gate, s_up: f32 [E, f]; s_down: f32 [E, d].
 *   Other arguments, outputs and conventions as zmoe_moe_layer with dtype ZMOE_BF16.
 * Decode sizes only (T * k < 64 E, T * k <= 1024, d and f multiples of 256): one cooperative
 * launch streams the codes (half the bf16 bytes), expands them to f16 in tensor memory and runs
 * f16 x f16 tensor-core contractions with fp32 accumulation, so the layer input and the hidden
 * activations are carried in f16 there: values beyond f16's range (|v| > 65504) count a device
 * error.  Larger sizes return ZMOE_ERR_UNSUPPORTED.
 */
ZMOE_API zmoe_status zmoe_moe_layer_fp8(const void* x, const float* h, const float* gamma, float eps,
                                        const void* w_router, const float* logit_bias, const float* sel_bias,
                                        const uint8_t* q_gate, const float* s_gate, const uint8_t* q_up,
                                        const float* s_up, const uint8_t* q_down, const float* s_down, int T, int d,
                                        int f, int E, int k, float* y, int32_t* expert_idx, float* gates,
                                        float* margin, void* x_norm, void* workspace, size_t ws_bytes,
                                        zmoe_stream_t stream);

/* Bytes of workspace zmoe_output_heads needs (T tokens, N codebooks). */
ZMOE_API size_t zmoe_output_heads_workspace_size(int T, int N);

/*
 * Output heads over the codebooks and the greedy next frame ([DIGEST] items 1 and 5: the decoder
 * predicts the next frame Y[t+1, n] of the 9 delay-patterned DAC codebooks):
 *   x = RMSNorm(h[t]) * gamma (gamma NULL: x = h[t]), rounded to `dtype`;
 *   logits[t, n, v] = sum_c w_heads[n, v, c] x[c]   (fp32 accumulation, one bias-free head per codebook);
 *   ids[t, n] = argmax_v logits[t, n, v], ties -> the lower id (-1, with a device error, only when
 *   every logit of that (t, n) is NaN).
 *   h: f32 [T, d]; gamma: f32 [d] or NULL; w_heads: [N, V, d] of `dtype`; ids: int32 [T, N];
 *   logits: f32 [T, N, V] or NULL; x_out: [T, d] of `dtype` or NULL (the rounded input).
 *   The weights are streamed once per 8 tokens.  d % 8 == 0, w_heads 16-byte aligned; workspace:
 *   zmoe_output_heads_workspace_size() bytes.  The pages give no head formula: the final norm and
 *   the bias-free linear heads are the plain pre-norm-transformer reading.
 */
ZMOE_API zmoe_status zmoe_output_heads(const float* h, const float* gamma, float eps, const void* w_heads,
                                       zmoe_dtype dtype, int T, int N, int V, int d, int32_t* ids, float* logits,
                                       void* x_out, void* workspace, size_t ws_bytes, zmoe_stream_t stream);

/*
 * Speaker-embedding prefix row ([DIGEST] item 3: the LDA-reduced speaker embedding is projected to
 * the model width and placed at position 0 of the decoder input):
 *   out[b] = W_spk e[b] + b_spk    (fp32 accumulation)
 *   e: f32 [B, n_in] (n_in = 1024 in ZONOS2); w_spk: [d, n_in] of `dtype`; b_spk: f32 [d] or NULL;
 *   out: f32 [B, d].  n_in % 8 == 0, w_spk 16-byte aligned.
 */
ZMOE_API zmoe_status zmoe_speaker_prefix(const float* e, const void* w_spk, zmoe_dtype dtype, const float* b_spk,
                                         int B, int d, int n_in, float* out, zmoe_stream_t stream);

/* Bytes of workspace zmoe_moe_layer_f16h needs. */
ZMOE_API size_t zmoe_moe_layer_f16h_workspace_size(int T, int d, int f, int E, int k);

/*
 * zmoe_moe_layer (same arguments, bf16) with the prepared f16 down weights (zmoe_prepare_w_down_f16) in
 * place of w_down, for prefill-size batches: pre-norm (with gamma), zmoe_route, zmoe_permute,
 * zmoe_grouped_swiglu_f16h, zmoe_combine, in order on `stream`.  The same layer as zmoe_moe_layer up to
 * h's rounding to f16 (~3e-3 of the output RMS at most on the skewed prefill layers).
 * d % 256 == 0, f % 256 == 0.
 */
ZMOE_API zmoe_status zmoe_moe_layer_f16h(const void* x, const float* h, const float* gamma, float eps,
                                         const void* w_router, const float* logit_bias, const float* sel_bias,
                                         const void* w_gate, const void* w_up, const void* w_down_f16,
                                         const float* down_scale, int T, int d, int f, int E, int k, float* y,
                                         int32_t* expert_idx, float* gates, float* margin, void* x_norm,
                                         void* workspace, size_t ws_bytes, zmoe_stream_t stream);

/* Bytes of workspace zmoe_moe_layer_w8a8 needs. */
ZMOE_API size_t zmoe_moe_layer_w8a8_workspace_size(int T, int d, int f, int E, int k);

/*
 * Where zmoe_moe_layer_w8a8 leaves its intermediates in the workspace (byte offsets, for inspection
 * after the call): offsets[0..9] = counts int32 [E], offsets int32 [E + 1], perm int32 [T k], inv_perm
 * int32 [T, k], the token rows' codes uint8 [T k, d] and scales f32 [T k], h f16 [T k, f], h's codes
 * uint8 [T k, f] and scales f32 [T k], y_perm f32 [T k, d] (rows in expert order).  n >= 10.
 */
ZMOE_API zmoe_status zmoe_moe_layer_w8a8_workspace_layout(int T, int d, int f, int E, int k, size_t* offsets, int n);

/*
 * The MoE layer in W8A8 fp8 for prefill-size batches ([COOKBOOK] Benchmark Results: the served ZONOS2
 * runs fp8; the reading is the common fp8 serving scheme with dynamic per-token activation scales).
 * Expert weights as in zmoe_moe_layer_fp8 (E4M3 codes, one fp32 scale per row: w = code * scale);
 * router in bf16.  Each row entering an expert GEMM -- the permuted token row, then the hidden row h --
 * is quantized per token: s = max|row| / 448 (fp32; 1 for an all-zero row), codes = the E4M3 value
 * nearest row x fp32(1 / s) (each product rounded to fp32; ties to even, saturating at 448).  The GEMMs run on tcgen05 kind::f8f6f4 (CTA pairs);
 * their fp32 sums are multiplied by the token scale and the weight row's scale; h is held in f16 between
 * the GEMMs (an |h| beyond 65504 counts a device error) and quantized from that.
 *   y[t] = h[t] + sum_i gate[t, i] * down_e( Q(silu(gate_e(Q(x[t]))) * up_e(Q(x[t]))) )   (h = 0 if NULL)
 * Arguments as zmoe_moe_layer_fp8 (x or h with gamma: bf16 / f32; the codes and the scale arrays 16-byte
 * aligned); any T (built for >= 64 rows per expert on average); d % 256 == 0, f % 256 == 0.
 */
ZMOE_API zmoe_status zmoe_moe_layer_w8a8(const void* x, const float* h, const float* gamma, float eps,
                                         const void* w_router, const float* logit_bias, const float* sel_bias,
                                         const uint8_t* q_gate, const float* s_gate, const uint8_t* q_up,
                                         const float* s_up, const uint8_t* q_down, const float* s_down, int T, int d,
                                         int f, int E, int k, float* y, int32_t* expert_idx, float* gates,
                                         float* margin, void* x_norm, void* workspace, size_t ws_bytes,
                                         zmoe_stream_t stream);

/* One layer of zmoe_decode_stack (bf16 weights, the layouts of zmoe_moe_layer). */
typedef struct zmoe_stack_layer {
  const void* w_router;     /* bf16 [E, d]; NULL only for a dense FFN layer (E == 1, k == 1: gate 1) */
  const float* logit_bias;  /* [E] or NULL: enters the gates and the selection */
  const float* sel_bias;    /* [E] or NULL: selection only */
  const float* gamma;       /* [d] the layer's pre-norm gain */
  const void* w_gate;       /* bf16 [E, f, d] */
  const void* w_up;         /* bf16 [E, f, d] */
  const void* w_down;       /* bf16 [E, d, f] */
  int E;                    /* experts, 1..64 */
  int k;                    /* experts per token, 1 or 2, <= E */
} zmoe_stack_layer;

/* Bytes of workspace zmoe_decode_stack needs for layers of at most E_max experts; 0 when these
 * sizes are not supported (see the limits below). */
ZMOE_API size_t zmoe_decode_stack_workspace_size(int n_layers, int d, int f, int E_max);

/*
 * The batch-1 decode stack in one call ([DIGEST] item 5: the decoder input is the RMSNorm of the
 * summed embeddings of the codebook frame; the FFN side of the decoder is a stack of pre-norm
 * residual blocks, dense or MoE, top-1 and top-2 in the last MoE layer; [ROUTING] section 2.1).
 * One token (T = 1):
 *   if ids:  h = RMSNorm(sum_j tables[j, ids[j]]) * gamma0     (fp32 sum, as zmoe_embed_sum_rmsnorm)
 *   for l < n_layers:  x = bf16(RMSNorm(h) * layers[l].gamma)
 *                      h = h + sum_{i<k} gate_i * FFN_{e_i}(x)  (router, top-k and gates as zmoe_route;
 *                                                                a dense layer: expert 0, gate 1)
 *   ids: int32 [N] or NULL (then h holds the stack input on entry); tables: bf16 [N, V, d]; gamma0:
 *   f32 [d]; h: f32 [d], in place (the final residual stream on return).
 *   Optional outputs (NULL to skip): layer_idx int32 [n_layers, 2] and layer_gates f32 [n_layers, 2]
 *   (the chosen experts and gates of each layer in slot order; -1 / 0 past k), layer_h f32
 *   [n_layers, d] (h entering each layer), layer_x bf16 [n_layers, d] (each layer's routed input).
 *   One persistent cooperative launch over all SMs (plus a 256-byte memset of the workspace): every
 *   CTA repeats the pre-norm and routing, the weights stream through shared memory, two grid
 *   barriers per layer.  Same arithmetic as n_layers zmoe_moe_layer calls with T = 1 (fp32 sums in a
 *   fixed order; the router's summation order differs, so ids can differ only on near-ties).
 *   Limits: n_layers <= 32, d % 8 == 0, d <= 4096, f % 8 == 0, N <= 32, at most 64 of the d rows
 *   per SM, and the per-CTA buffers must fit one SM's shared memory: a 4-slot ring of weight blocks
 *   (a block = as many 2 d- or 2 f-byte rows as fit 32 KB, 1 to 7), max(E d 2, 8 f) bytes for the
 *   router rows and then the chosen experts' h, 8 d bytes of gain and x, and ~2 KB of control.
 *   d = 2048, f = 3072, E = 16 fits; larger sizes return ZMOE_ERR_UNSUPPORTED.  Ids outside [0, V)
 *   count a device error and contribute nothing.
 */
ZMOE_API zmoe_status zmoe_decode_stack(const zmoe_stack_layer* layers, int n_layers, int d, int f, float eps,
                                       const int32_t* ids, const void* tables, const float* gamma0, int N, int V,
                                       float* h, int32_t* layer_idx, float* layer_gates, float* layer_h,
                                       void* layer_x, void* workspace, size_t ws_bytes, zmoe_stream_t stream);

/*
 * Reads and clears the device error counters of the current device.  Synchronises
 * `stream` (and the device) first.  *count = data errors (ids or indices out of range)
 * plus bounded device-side waits that gave up, since the last read.  Returns
 * ZMOE_ERR_TIMEOUT when any wait gave up, else ZMOE_ERR_DEVICE_CHECK when *count > 0,
 * else ZMOE_OK.
 */
ZMOE_API zmoe_status zmoe_get_device_errors(zmoe_stream_t stream, uint32_t* count);

/*
 * Fault injection for tests of the timeout path (no counterpart on the pages; failure detection of
 * the library itself).  With extra > 0, every later launch of the stream-K decode kernels
 * (zmoe_moe_layer and zmoe_moe_layer_fp8 at decode sizes, zmoe_grouped_swiglu below 64 rows per
 * expert) makes its phase-A -> phase-B hand-off wait for `extra` more finished phase-A units than
 * exist, giving up after limit_ns (in [1 us, 2 s]) instead of the usual 2 s.  The wait then runs
 * out: each CTA counts a timeout, stops, waits (bounded) for its own copies and MMAs, frees its
 * tensor memory and returns, and zmoe_get_device_errors() reports ZMOE_ERR_TIMEOUT.  The outputs of
 * such a launch are undefined.  zmoe_debug_inject_timeout(0, 0) restores normal operation.  The
 * setting is process-wide and read when a call launches; for tests only.
 */
ZMOE_API zmoe_status zmoe_debug_inject_timeout(uint32_t extra, uint64_t limit_ns);

#ifdef __cplusplus
}
#endif

#endif /* ZMOE_H */
