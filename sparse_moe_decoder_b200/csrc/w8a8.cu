// The MoE layer in W8A8 fp8 for prefill-size batches: E4M3 expert weights with one fp32 scale per row
// (w = code * scale) and E4M3 activations with one dynamic scale per token.
//
// The ZONOS2 serving stack runs the model in fp8 (ZONOS2 page of the sglang-omni cookbook, "Benchmark
// Results").  Reading taken for prefill sizes: the common fp8 serving scheme with dynamic activation
// quantization: each row entering an expert GEMM (the permuted token row, then the hidden row h) gets
//   s = max|row| / 448  (fp32; 1 for an all-zero row),   codes = E4M3 nearest row x fp32(1 / s) (ties
//   to even, saturating at 448; one correctly rounded reciprocal per row, one product per element),
// and the tensor cores run kind::f8f6f4 at twice the bf16 rate; the fp32 sums are multiplied by the row's
// token scale and the weight row's scale.  h is held in f16 between the two GEMMs (the first GEMM's
// epilogue also records each row's max |h|), then quantized per token.
//
// Order on the stream: [pre-norm] -> router -> permutation indices -> gather + quantize of the token
// rows -> gate/up GEMM (E4M3, CTA pairs) -> h quantization -> down GEMM (E4M3) -> combine.
#include <cuda_fp8.h>

#include "common.cuh"

namespace zmoe {

zmoe_status permute_indices(const int32_t* expert_idx, int T, int E, int k, int32_t* counts, int32_t* offsets,
                            int32_t* perm, int32_t* inv_perm, void* workspace, size_t ws_bytes, cudaStream_t s);
zmoe_status grouped_gateup_tc_e4m3(const uint8_t* xq, const float* sx, const int32_t* offsets, int M_total,
                                   const uint8_t* q_gate, const float* s_gate, const uint8_t* q_up, const float* s_up,
                                   int E, int d, int f, uint16_t* h16, unsigned int* amax, cudaStream_t s);
zmoe_status grouped_down_tc_e4m3(const uint8_t* hq, const float* sh, const int32_t* offsets, int M_total,
                                 const uint8_t* q_down, const float* s_down, int E, int d, int f, float* y_perm,
                                 cudaStream_t s);
bool grouped_swiglu_tc_supported(int d, int f);

namespace {

constexpr int kThreads = 256;

// Two values -> two E4M3 codes (round to nearest even, saturating at +-448), the first in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  return static_cast<uint16_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// The per-token scale of a row whose largest magnitude is amax.
__device__ __forceinline__ float token_scale(float amax) { return amax > 0.f ? __fdiv_rn(amax, 448.f) : 1.f; }

// 8 values (fp32) multiplied by r = fp32(1 / s) and encoded: 8 codes in a uint2, the first value in the
// lowest byte.
__device__ __forceinline__ uint2 encode8(const float* v, float r) {
  uint32_t w[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const uint16_t a = e4m3x2(__fmul_rn(v[4 * i], r), __fmul_rn(v[4 * i + 1], r));
    const uint16_t b = e4m3x2(__fmul_rn(v[4 * i + 2], r), __fmul_rn(v[4 * i + 3], r));
    w[i] = static_cast<uint32_t>(a) | (static_cast<uint32_t>(b) << 16);
  }
  return make_uint2(w[0], w[1]);
}

constexpr int kRowChunks = 12;   // a row of up to 12 x 256 elements stays in registers (8 per lane per chunk)

// xq[r] = E4M3(x[perm[r]] x fp32(1 / sx[r])), sx[r] = max|x[perm[r]]| / 448, one warp per permuted row
// (the row is read once into registers when d <= 256 kRowChunks).
__global__ void __launch_bounds__(kThreads) gather_quantize_kernel(const uint16_t* __restrict__ x,
                                                                    const int32_t* __restrict__ perm,
                                                                    const int32_t* __restrict__ offsets, int E, int d,
                                                                    uint8_t* __restrict__ xq, float* __restrict__ sx) {
  const int lane = threadIdx.x & 31;
  const long long rows = offsets[E];
  const long long warps = static_cast<long long>(gridDim.x) * (kThreads / 32);
  const bool in_regs = d <= 256 * kRowChunks;
  for (long long r = blockIdx.x * static_cast<long long>(kThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const uint16_t* src = x + static_cast<size_t>(perm[r]) * d;
    uint4 raw[kRowChunks];
    float amax = 0.f;
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kRowChunks; ++j) {
        const int c = lane * 8 + j * 256;
        raw[j] = c < d ? __ldg(reinterpret_cast<const uint4*>(src + c)) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int j = 0; j < kRowChunks; ++j) {
        float v[8];
        unpack_bf16x8(raw[j], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    } else {
      for (int c = lane * 8; c < d; c += 256) {
        float v[8];
        unpack_bf16x8(*reinterpret_cast<const uint4*>(src + c), v);
#pragma unroll
        for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(v[i]));
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = token_scale(amax), rs = __frcp_rn(s);
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kRowChunks; ++j) {
        const int c = lane * 8 + j * 256;
        if (c < d) {
          float v[8];
          unpack_bf16x8(raw[j], v);
          *reinterpret_cast<uint2*>(xq + static_cast<size_t>(r) * d + c) = encode8(v, rs);
        }
      }
    } else {
      for (int c = lane * 8; c < d; c += 256) {
        float v[8];
        unpack_bf16x8(*reinterpret_cast<const uint4*>(src + c), v);
        *reinterpret_cast<uint2*>(xq + static_cast<size_t>(r) * d + c) = encode8(v, rs);
      }
    }
    if (lane == 0) sx[r] = s;
  }
}

// hq[r] = E4M3(h16[r] x fp32(1 / sh[r])), sh[r] = amax[r] / 448 (amax: bits of max |h16[r]|), one warp
// per row.
__global__ void __launch_bounds__(kThreads) quantize_h_kernel(const uint16_t* __restrict__ h16,
                                                               const unsigned int* __restrict__ amax,
                                                               const int32_t* __restrict__ offsets, int E, int f,
                                                               uint8_t* __restrict__ hq, float* __restrict__ sh) {
  const int lane = threadIdx.x & 31;
  const long long rows = offsets[E];
  const long long warps = static_cast<long long>(gridDim.x) * (kThreads / 32);
  for (long long r = blockIdx.x * static_cast<long long>(kThreads / 32) + (threadIdx.x >> 5); r < rows; r += warps) {
    const float s = token_scale(__uint_as_float(amax[r])), rs = __frcp_rn(s);
    const uint16_t* src = h16 + static_cast<size_t>(r) * f;
    for (int c = lane * 8; c < f; c += 256) {
      const uint4 raw = *reinterpret_cast<const uint4*>(src + c);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      float v[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        v[2 * i] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] & 0xFFFFu)));
        v[2 * i + 1] = __half2float(__ushort_as_half(static_cast<unsigned short>(w[i] >> 16)));
      }
      *reinterpret_cast<uint2*>(hq + static_cast<size_t>(r) * f + c) = encode8(v, rs);
    }
    if (lane == 0) sh[r] = s;
  }
}

size_t a256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct W8Ws {
  size_t x_norm, idx, gates, counts, offsets, perm, inv_perm, perm_ws, xq, sx, h16, amax, hq, sh, y_perm, total;
  size_t perm_ws_bytes;
};

W8Ws w8_ws(int T, int E, int d, int f, int k) {
  W8Ws W{};
  const size_t n = static_cast<size_t>(T) * k;
  size_t o = 0;
  auto take = [&o](size_t bytes) {
    const size_t at = o;
    o = a256(o + bytes);
    return at;
  };
  W.x_norm = take(static_cast<size_t>(T) * d * 2);
  W.idx = take(n * 4);
  W.gates = take(n * 4);
  W.counts = take(static_cast<size_t>(E) * 4);
  W.offsets = take(static_cast<size_t>(E + 1) * 4);
  W.perm = take(n * 4);
  W.inv_perm = take(n * 4);
  W.perm_ws_bytes = zmoe_permute_workspace_size(T, E, k);
  W.perm_ws = take(W.perm_ws_bytes);
  W.xq = take(n * d);
  W.sx = take(n * 4);
  W.h16 = take(n * f * 2);
  W.amax = take(n * 4);
  W.hq = take(n * f);
  W.sh = take(n * 4);
  W.y_perm = take(n * d * 4);
  W.total = o;
  return W;
}

int rows_grid(long long rows) {
  long long g = (rows + kThreads / 32 - 1) / (kThreads / 32);
  const long long cap = static_cast<long long>(num_sms()) * 8;
  return static_cast<int>(g < 1 ? 1 : (g > cap ? cap : g));
}

}  // namespace
}  // namespace zmoe

extern "C" {

size_t zmoe_moe_layer_w8a8_workspace_size(int T, int d, int f, int E, int k) {
  using namespace zmoe;
  if (T <= 0 || d < 1 || f < 1 || E < 1 || E > 64 || (k != 1 && k != 2)) return 0;
  return w8_ws(T, E, d, f, k).total;
}

zmoe_status zmoe_moe_layer_w8a8_workspace_layout(int T, int d, int f, int E, int k, size_t* offsets, int n) {
  using namespace zmoe;
  ZMOE_REQUIRE(offsets && n >= 10, "zmoe_moe_layer_w8a8_workspace_layout: needs 10 offsets");
  ZMOE_REQUIRE(T > 0 && d > 0 && f > 0 && E >= 1 && E <= 64 && (k == 1 || k == 2),
               "zmoe_moe_layer_w8a8_workspace_layout: bad sizes");
  const W8Ws W = w8_ws(T, E, d, f, k);
  const size_t o[10] = {W.counts, W.offsets, W.perm, W.inv_perm, W.xq, W.sx, W.h16, W.hq, W.sh, W.y_perm};
  for (int i = 0; i < 10; ++i) offsets[i] = o[i];
  return ZMOE_OK;
}

zmoe_status zmoe_moe_layer_w8a8(const void* x, const float* h, const float* gamma, float eps, const void* w_router,
                                const float* logit_bias, const float* sel_bias, const uint8_t* q_gate,
                                const float* s_gate, const uint8_t* q_up, const float* s_up, const uint8_t* q_down,
                                const float* s_down, int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                                float* gates, float* margin, void* x_norm, void* workspace, size_t ws_bytes,
                                zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_moe_layer_w8a8");
  using namespace zmoe;
  ZMOE_REQUIRE(T >= 0, "zmoe_moe_layer_w8a8: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_moe_layer_w8a8: E must be in [1, 64]");
  ZMOE_REQUIRE((k == 1 || k == 2) && k <= E, "zmoe_moe_layer_w8a8: k must be 1 or 2 and <= E");
  ZMOE_REQUIRE(d >= 256 && d % 256 == 0 && f >= 256 && f % 256 == 0,
               "zmoe_moe_layer_w8a8: d and f must be multiples of 256");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE(static_cast<long long>(T) * k * (d > f ? d : f) <= 0x7fffffffLL,
               "zmoe_moe_layer_w8a8: T * k * max(d, f) overflows int32");
  ZMOE_REQUIRE((w_router || E == 1) && q_gate && s_gate && q_up && s_up && q_down && s_down && y,
               "zmoe_moe_layer_w8a8: NULL pointer (w_router may be NULL only when E == 1)");
  ZMOE_REQUIRE(gamma ? h != nullptr : x != nullptr, "zmoe_moe_layer_w8a8: needs x, or h with gamma");
  ZMOE_REQUIRE((!x || aligned16(x)) && (!h || aligned16(h)) && aligned16(y) && (!w_router || aligned16(w_router)) &&
                   aligned16(q_gate) && aligned16(q_up) && aligned16(q_down) && (!x_norm || aligned16(x_norm)) &&
                   (!gamma || aligned16(gamma)) && aligned16(s_gate) && aligned16(s_up) && aligned16(s_down),
               "zmoe_moe_layer_w8a8: pointers must be 16-byte aligned");
  if (!grouped_swiglu_tc_supported(d, f))
    return fail(ZMOE_ERR_UNSUPPORTED, "zmoe_moe_layer_w8a8: no tensor-core kernel for this d, f");
  const size_t need = zmoe_moe_layer_w8a8_workspace_size(T, d, f, E, k);
  if (!workspace || ws_bytes < need)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                "zmoe_moe_layer_w8a8: workspace smaller than zmoe_moe_layer_w8a8_workspace_size()");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const W8Ws W = w8_ws(T, E, d, f, k);
  unsigned char* w = static_cast<unsigned char*>(workspace);
  const int M = T * k;
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
  auto* counts = reinterpret_cast<int32_t*>(w + W.counts);
  auto* offsets = reinterpret_cast<int32_t*>(w + W.offsets);
  auto* perm = reinterpret_cast<int32_t*>(w + W.perm);
  auto* inv = reinterpret_cast<int32_t*>(w + W.inv_perm);
  st = permute_indices(idx, T, E, k, counts, offsets, perm, inv, w + W.perm_ws, W.perm_ws_bytes, s);
  if (st != ZMOE_OK) return st;
  auto* xq = reinterpret_cast<uint8_t*>(w + W.xq);
  auto* sx = reinterpret_cast<float*>(w + W.sx);
  gather_quantize_kernel<<<rows_grid(M), kThreads, 0, s>>>(static_cast<const uint16_t*>(xin), perm, offsets, E, d, xq,
                                                            sx);
  if ((st = check_launch("zmoe_moe_layer_w8a8 (quantize x)")) != ZMOE_OK) return st;
  auto* amax = reinterpret_cast<unsigned int*>(w + W.amax);
  if (cudaMemsetAsync(amax, 0, static_cast<size_t>(M) * 4, s) != cudaSuccess)
    return check_launch("zmoe_moe_layer_w8a8: clearing");
  auto* h16 = reinterpret_cast<uint16_t*>(w + W.h16);
  st = grouped_gateup_tc_e4m3(xq, sx, offsets, M, q_gate, s_gate, q_up, s_up, E, d, f, h16, amax, s);
  if (st != ZMOE_OK) return st;
  auto* hq = reinterpret_cast<uint8_t*>(w + W.hq);
  auto* sh = reinterpret_cast<float*>(w + W.sh);
  quantize_h_kernel<<<rows_grid(M), kThreads, 0, s>>>(h16, amax, offsets, E, f, hq, sh);
  if ((st = check_launch("zmoe_moe_layer_w8a8 (quantize h)")) != ZMOE_OK) return st;
  float* yp = reinterpret_cast<float*>(w + W.y_perm);
  st = grouped_down_tc_e4m3(hq, sh, offsets, M, q_down, s_down, E, d, f, yp, s);
  if (st != ZMOE_OK) return st;
  return zmoe_combine(yp, inv, g, h, T, d, k, y, stream);
}

}  // extern "C"
