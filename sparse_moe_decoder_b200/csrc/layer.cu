// zmoe_moe_layer: one sparse MoE layer of the decoder, optionally with its pre-norm:
//   x    = RMSNorm(h) * gamma, rounded to the compute dtype    (when gamma is given; else x is the input)
//   y[t] = h[t] + sum_{i < k} gate[t, i] * FFN_{e(t, i)}(x[t])  (h = 0 when not given)
// ZONOS2 digest items 5-6 (sparse MoE FFN, top-1 / top-2 routing, RMSNorm), the telknet.cc article
// on ZONOS2, section 2.1 (router, gate-weighted sum of the chosen experts).
//
// A few tokens (bf16, T * k <= 4) run as one cooperative launch of CUDA-core matrix-vector products
// without split-k (tiny_layer.cu).  Decode sizes (bf16, T * k < 64 E and T * k <= 1024) run as ONE
// cooperative launch (decode_tc.cu: pre-norm + router, grid barrier, dispatch, grid barrier,
// stream-K SwiGLU with the combine in its epilogue).  Every other size runs the separate entry points
// in order: zmoe_rmsnorm, zmoe_route, zmoe_permute, zmoe_grouped_swiglu, zmoe_combine.
#include "common.cuh"

namespace zmoe {

bool moe_layer_fused_supported(int T, int E, int d, int f, int k);
size_t moe_layer_fused_workspace(int T, int E, int d, int f, int k);
zmoe_status moe_layer_fused(const uint16_t* x, const float* h_in, const float* gamma, float eps, const uint16_t* w_r,
                            const float* logit_bias, const float* sel_bias, const void* w_gate, const void* w_up,
                            const void* w_down, int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                            float* gates, float* margin, uint16_t* x_norm_out, void* ws, cudaStream_t s,
                            const float* s_gate, const float* s_up, const float* s_down);

bool moe_layer_tiny_supported(int T, int E, int d, int f, int k);
size_t moe_layer_tiny_workspace(int T, int f, int k);
zmoe_status moe_layer_tiny(const uint16_t* x, const float* h_in, const float* gamma, float eps, const uint16_t* w_r,
                           const float* logit_bias, const float* sel_bias, const uint16_t* w_gate, const uint16_t* w_up,
                           const uint16_t* w_down, int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                           float* gates, float* margin, uint16_t* x_norm, void* ws, cudaStream_t s);

namespace {

bool use_tiny(int T, int E, int d, int f, int k, zmoe_dtype dtype) {
  return dtype == ZMOE_BF16 && moe_layer_tiny_supported(T, E, d, f, k);
}

// Rows per expert below which the fused decode launch is used (the grouped SwiGLU's own
// decode / prefill threshold).
constexpr int kFusedRowsPerExpert = 64;

bool use_fused(int T, int E, int d, int f, int k, zmoe_dtype dtype) {
  return dtype == ZMOE_BF16 && static_cast<long long>(T) * k < static_cast<long long>(kFusedRowsPerExpert) * E &&
         moe_layer_fused_supported(T, E, d, f, k);
}

size_t a256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct SeqWs {
  size_t x_norm, idx, gates, counts, offsets, perm, inv_perm, x_perm, h, y_perm, perm_ws, ffn_ws, total;
  size_t perm_ws_bytes, ffn_ws_bytes;
};

SeqWs seq_ws(int T, int E, int d, int f, int k, zmoe_dtype dtype) {
  SeqWs W{};
  const size_t n = static_cast<size_t>(T) * k, es = dtype_size(dtype);
  size_t o = 0;
  auto take = [&o](size_t bytes) {
    const size_t at = o;
    o = a256(o + bytes);
    return at;
  };
  W.x_norm = take(static_cast<size_t>(T) * d * es);
  W.idx = take(n * 4);
  W.gates = take(n * 4);
  W.counts = take(static_cast<size_t>(E) * 4);
  W.offsets = take(static_cast<size_t>(E + 1) * 4);
  W.perm = take(n * 4);
  W.inv_perm = take(n * 4);
  W.x_perm = take(n * d * es);
  W.h = take(dtype == ZMOE_BF16 ? n * 2 * f * 2 : n * f * 4);
  W.y_perm = take(n * d * 4);
  W.perm_ws_bytes = zmoe_permute_workspace_size(T, E, k);
  W.perm_ws = take(W.perm_ws_bytes);
  W.ffn_ws_bytes = zmoe_grouped_swiglu_workspace_size(static_cast<int>(n), E, d, f, dtype);
  W.ffn_ws = take(W.ffn_ws_bytes);
  W.total = o;
  return W;
}

}  // namespace
}  // namespace zmoe

extern "C" {

size_t zmoe_moe_layer_workspace_size(int T, int d, int f, int E, int k, zmoe_dtype dtype) {
  using namespace zmoe;
  if (T < 0 || d < 1 || f < 1 || E < 1 || E > 64 || (k != 1 && k != 2) || !dtype_ok(dtype)) return 0;
  if (T == 0) return 0;
  if (use_tiny(T, E, d, f, k, dtype)) return moe_layer_tiny_workspace(T, f, k);
  if (use_fused(T, E, d, f, k, dtype)) return moe_layer_fused_workspace(T, E, d, f, k);
  return seq_ws(T, E, d, f, k, dtype).total;
}

zmoe_status zmoe_moe_layer(const void* x, const float* h, const float* gamma, float eps, const void* w_router,
                           const float* logit_bias, const float* sel_bias, const void* w_gate, const void* w_up,
                           const void* w_down, zmoe_dtype dtype, int T, int d, int f, int E, int k, float* y,
                           int32_t* expert_idx, float* gates, float* margin, void* x_norm, void* workspace,
                           size_t ws_bytes, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_moe_layer");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_moe_layer: bad dtype");
  ZMOE_REQUIRE(T >= 0, "zmoe_moe_layer: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_moe_layer: E must be in [1, 64]");
  ZMOE_REQUIRE((k == 1 || k == 2) && k <= E, "zmoe_moe_layer: k must be 1 or 2 and <= E");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0 && f >= 8 && f % 8 == 0, "zmoe_moe_layer: d and f must be multiples of 8");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE((w_router || E == 1) && w_gate && w_up && w_down && y,
               "zmoe_moe_layer: NULL pointer (w_router may be NULL only when E == 1)");
  ZMOE_REQUIRE(gamma ? h != nullptr : x != nullptr, "zmoe_moe_layer: needs x, or h with gamma");
  ZMOE_REQUIRE((!x || aligned16(x)) && (!h || aligned16(h)) && aligned16(y) && (!w_router || aligned16(w_router)) &&
                   aligned16(w_gate) && aligned16(w_up) && aligned16(w_down) && (!x_norm || aligned16(x_norm)) &&
                   (!gamma || aligned16(gamma)),
               "zmoe_moe_layer: pointers must be 16-byte aligned");
  const size_t need = zmoe_moe_layer_workspace_size(T, d, f, E, k, dtype);
  if (!workspace || ws_bytes < need)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL, "zmoe_moe_layer: workspace smaller than zmoe_moe_layer_workspace_size()");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (use_tiny(T, E, d, f, k, dtype))
    return moe_layer_tiny(static_cast<const uint16_t*>(x), h, gamma, eps, static_cast<const uint16_t*>(w_router),
                          logit_bias, sel_bias, static_cast<const uint16_t*>(w_gate), static_cast<const uint16_t*>(w_up),
                          static_cast<const uint16_t*>(w_down), T, d, f, E, k, y, expert_idx, gates, margin,
                          static_cast<uint16_t*>(x_norm), workspace, s);
  if (use_fused(T, E, d, f, k, dtype))
    return moe_layer_fused(static_cast<const uint16_t*>(x), h, gamma, eps, static_cast<const uint16_t*>(w_router),
                           logit_bias, sel_bias, w_gate, w_up, w_down, T, d, f, E, k, y, expert_idx, gates, margin,
                           static_cast<uint16_t*>(x_norm), workspace, s, nullptr, nullptr, nullptr);

  const SeqWs W = seq_ws(T, E, d, f, k, dtype);
  unsigned char* w = static_cast<unsigned char*>(workspace);
  const void* xin = x;
  if (gamma) {
    void* xn = x_norm ? x_norm : static_cast<void*>(w + W.x_norm);
    zmoe_status st = zmoe_rmsnorm(h, ZMOE_F32, gamma, eps, T, d, xn, dtype, stream);
    if (st != ZMOE_OK) return st;
    xin = xn;
  }
  int32_t* idx = expert_idx ? expert_idx : reinterpret_cast<int32_t*>(w + W.idx);
  float* g = gates ? gates : reinterpret_cast<float*>(w + W.gates);
  zmoe_status st = zmoe_route(xin, w_router, dtype, logit_bias, sel_bias, T, d, E, k, idx, g, margin, stream);
  if (st != ZMOE_OK) return st;
  int32_t* inv = reinterpret_cast<int32_t*>(w + W.inv_perm);
  st = zmoe_permute(idx, xin, dtype, T, d, E, k, reinterpret_cast<int32_t*>(w + W.counts),
                    reinterpret_cast<int32_t*>(w + W.offsets), reinterpret_cast<int32_t*>(w + W.perm), inv,
                    w + W.x_perm, w + W.perm_ws, W.perm_ws_bytes, stream);
  if (st != ZMOE_OK) return st;
  float* yp = reinterpret_cast<float*>(w + W.y_perm);
  st = zmoe_grouped_swiglu(w + W.x_perm, reinterpret_cast<int32_t*>(w + W.offsets), T * k, w_gate, w_up, w_down, dtype,
                           E, d, f, w + W.h, yp, w + W.ffn_ws, W.ffn_ws_bytes, stream);
  if (st != ZMOE_OK) return st;
  (void)s;
  return zmoe_combine(yp, inv, g, h, T, d, k, y, stream);
}

size_t zmoe_moe_layer_fp8_workspace_size(int T, int d, int f, int E, int k) {
  using namespace zmoe;
  if (T <= 0 || d < 1 || f < 1 || E < 1 || E > 64 || (k != 1 && k != 2) || !moe_layer_fused_supported(T, E, d, f, k))
    return 0;
  return moe_layer_fused_workspace(T, E, d, f, k);
}

zmoe_status zmoe_moe_layer_fp8(const void* x, const float* h, const float* gamma, float eps, const void* w_router,
                               const float* logit_bias, const float* sel_bias, const uint8_t* q_gate,
                               const float* s_gate, const uint8_t* q_up, const float* s_up, const uint8_t* q_down,
                               const float* s_down, int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                               float* gates, float* margin, void* x_norm, void* workspace, size_t ws_bytes,
                               zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_moe_layer_fp8");
  using namespace zmoe;
  ZMOE_REQUIRE(T >= 0, "zmoe_moe_layer_fp8: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_moe_layer_fp8: E must be in [1, 64]");
  ZMOE_REQUIRE((k == 1 || k == 2) && k <= E, "zmoe_moe_layer_fp8: k must be 1 or 2 and <= E");
  ZMOE_REQUIRE(d % 256 == 0 && f % 256 == 0 && d > 0 && f > 0, "zmoe_moe_layer_fp8: d and f must be multiples of 256");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE((w_router || E == 1) && q_gate && s_gate && q_up && s_up && q_down && s_down && y,
               "zmoe_moe_layer_fp8: NULL pointer (w_router may be NULL only when E == 1)");
  ZMOE_REQUIRE(gamma ? h != nullptr : x != nullptr, "zmoe_moe_layer_fp8: needs x, or h with gamma");
  ZMOE_REQUIRE((!x || aligned16(x)) && (!h || aligned16(h)) && aligned16(y) && (!w_router || aligned16(w_router)) &&
                   aligned16(q_gate) && aligned16(q_up) && aligned16(q_down) && (!x_norm || aligned16(x_norm)) &&
                   (!gamma || aligned16(gamma)),
               "zmoe_moe_layer_fp8: pointers must be 16-byte aligned");
  if (!moe_layer_fused_supported(T, E, d, f, k) || static_cast<long long>(T) * k >= 64LL * E)
    return fail(ZMOE_ERR_UNSUPPORTED, "zmoe_moe_layer_fp8: decode sizes only (T * k < 64 E, T * k <= 1024)");
  const size_t need = zmoe_moe_layer_fp8_workspace_size(T, d, f, E, k);
  if (!workspace || ws_bytes < need)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                "zmoe_moe_layer_fp8: workspace smaller than zmoe_moe_layer_fp8_workspace_size()");
  clear_error();
  return moe_layer_fused(static_cast<const uint16_t*>(x), h, gamma, eps, static_cast<const uint16_t*>(w_router),
                         logit_bias, sel_bias, q_gate, q_up, q_down, T, d, f, E, k, y, expert_idx, gates, margin,
                         static_cast<uint16_t*>(x_norm), workspace, reinterpret_cast<cudaStream_t>(stream), s_gate,
                         s_up, s_down);
}

size_t zmoe_moe_layer_f16h_workspace_size(int T, int d, int f, int E, int k) {
  using namespace zmoe;
  if (T <= 0 || d < 1 || f < 1 || E < 1 || E > 64 || (k != 1 && k != 2)) return 0;
  return seq_ws(T, E, d, f, k, ZMOE_BF16).total;
}

zmoe_status zmoe_moe_layer_f16h(const void* x, const float* h, const float* gamma, float eps, const void* w_router,
                                const float* logit_bias, const float* sel_bias, const void* w_gate, const void* w_up,
                                const void* w_down_f16, const float* down_scale, int T, int d, int f, int E, int k,
                                float* y, int32_t* expert_idx, float* gates, float* margin, void* x_norm,
                                void* workspace, size_t ws_bytes, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_moe_layer_f16h");
  using namespace zmoe;
  ZMOE_REQUIRE(T >= 0, "zmoe_moe_layer_f16h: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_moe_layer_f16h: E must be in [1, 64]");
  ZMOE_REQUIRE((k == 1 || k == 2) && k <= E, "zmoe_moe_layer_f16h: k must be 1 or 2 and <= E");
  ZMOE_REQUIRE(d >= 256 && d % 256 == 0 && f >= 256 && f % 256 == 0,
               "zmoe_moe_layer_f16h: d and f must be multiples of 256");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE((w_router || E == 1) && w_gate && w_up && w_down_f16 && down_scale && y,
               "zmoe_moe_layer_f16h: NULL pointer (w_router may be NULL only when E == 1)");
  ZMOE_REQUIRE(gamma ? h != nullptr : x != nullptr, "zmoe_moe_layer_f16h: needs x, or h with gamma");
  ZMOE_REQUIRE((!x || aligned16(x)) && (!h || aligned16(h)) && aligned16(y) && (!w_router || aligned16(w_router)) &&
                   aligned16(w_gate) && aligned16(w_up) && aligned16(w_down_f16) && (!x_norm || aligned16(x_norm)) &&
                   (!gamma || aligned16(gamma)),
               "zmoe_moe_layer_f16h: pointers must be 16-byte aligned");
  const size_t need = zmoe_moe_layer_f16h_workspace_size(T, d, f, E, k);
  if (!workspace || ws_bytes < need)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                "zmoe_moe_layer_f16h: workspace smaller than zmoe_moe_layer_f16h_workspace_size()");
  clear_error();
  const SeqWs W = seq_ws(T, E, d, f, k, ZMOE_BF16);
  unsigned char* w = static_cast<unsigned char*>(workspace);
  const void* xin = x;
  if (gamma) {
    void* xn = x_norm ? x_norm : static_cast<void*>(w + W.x_norm);
    zmoe_status st = zmoe_rmsnorm(h, ZMOE_F32, gamma, eps, T, d, xn, ZMOE_BF16, stream);
    if (st != ZMOE_OK) return st;
    xin = xn;
  }
  int32_t* idx = expert_idx ? expert_idx : reinterpret_cast<int32_t*>(w + W.idx);
  float* g = gates ? gates : reinterpret_cast<float*>(w + W.gates);
  zmoe_status st = zmoe_route(xin, w_router, ZMOE_BF16, logit_bias, sel_bias, T, d, E, k, idx, g, margin, stream);
  if (st != ZMOE_OK) return st;
  int32_t* inv = reinterpret_cast<int32_t*>(w + W.inv_perm);
  st = zmoe_permute(idx, xin, ZMOE_BF16, T, d, E, k, reinterpret_cast<int32_t*>(w + W.counts),
                    reinterpret_cast<int32_t*>(w + W.offsets), reinterpret_cast<int32_t*>(w + W.perm), inv,
                    w + W.x_perm, w + W.perm_ws, W.perm_ws_bytes, stream);
  if (st != ZMOE_OK) return st;
  float* yp = reinterpret_cast<float*>(w + W.y_perm);
  st = zmoe_grouped_swiglu_f16h(w + W.x_perm, reinterpret_cast<int32_t*>(w + W.offsets), T * k, w_gate, w_up,
                                w_down_f16, down_scale, E, d, f, w + W.h, yp, stream);
  if (st != ZMOE_OK) return st;
  return zmoe_combine(yp, inv, g, h, T, d, k, y, stream);
}

}  // extern "C"
