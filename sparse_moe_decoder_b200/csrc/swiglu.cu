// zmoe_grouped_swiglu: per-expert SwiGLU over the permuted rows, and its fp32 kernels.
//
// ("GLU Variants Improve Transformer", ZONOS2 Technical Report "Builds on"; SiLU per the
// telknet.cc article on ZONOS2, section 2.1.)
//   h[r] = silu(W_gate[e] x[r]) * (W_up[e] x[r]);  y_perm[r] = W_down[e] h[r]
//
// Dispatch:
//   f32  -> plain fp32 FMA kernels (no TF32 anywhere: one thread per output, float4 loads).
//   bf16 -> rows per expert small (decode): one persistent stream-K launch on the tensor cores
//           with weights as the MMA's M and tokens as its N (swiglu_dec_tc.cu);
//           rows per expert large (prefill): tcgen05 / TMEM / TMA grouped GEMMs (swiglu_tc.cu).
//           Both keep h as a bf16 pair h_hi + h_lo ([M, 2f]) so that the second contraction
//           sees h to ~16 significant bits with bf16 tensor-core operands.
#include "common.cuh"

namespace zmoe {

zmoe_status grouped_swiglu_dec_tc(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                                  const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                                  float* y_perm, void* ws, cudaStream_t s);
size_t grouped_swiglu_dec_tc_workspace(int M_total, int E, int d, int f);
bool grouped_swiglu_dec_tc_supported(int d, int f);
zmoe_status grouped_swiglu_tc(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                              const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                              float* y_perm, void* ws, size_t ws_bytes, cudaStream_t s);
zmoe_status grouped_swiglu_tc_f16h(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                                   const uint16_t* w_up, const uint16_t* w_down_f16, const float* down_scale, int E,
                                   int d, int f, uint16_t* h, float* y_perm, cudaStream_t s);
size_t grouped_swiglu_tc_workspace(int M_total, int E, int d, int f);
bool grouped_swiglu_tc_supported(int d, int f);

namespace {

// Expert of permuted row m (E when m is past the last row).
__device__ __forceinline__ int expert_of_row(const int32_t* off, int E, int m) {
  int e = 0;
  while (e < E && off[e + 1] <= m) ++e;
  return e;
}

__device__ __forceinline__ float dot_f32(const float* __restrict__ a, const float* __restrict__ b, int n) {
  float acc = 0.f;
  const float4* a4 = reinterpret_cast<const float4*>(a);
  const float4* b4 = reinterpret_cast<const float4*>(b);
  for (int i = 0; i < n / 4; ++i) {
    const float4 u = __ldg(a4 + i), v = __ldg(b4 + i);
    acc = fmaf(u.x, v.x, acc);
    acc = fmaf(u.y, v.y, acc);
    acc = fmaf(u.z, v.z, acc);
    acc = fmaf(u.w, v.w, acc);
  }
  return acc;
}

__global__ void gateup_f32_kernel(const float* __restrict__ x, const int32_t* __restrict__ offsets, int E, int d,
                                  int f, const float* __restrict__ wg, const float* __restrict__ wu,
                                  float* __restrict__ h) {
  __shared__ int off[65];
  if (threadIdx.x <= E) off[threadIdx.x] = offsets[threadIdx.x];
  __syncthreads();
  const long long total = static_cast<long long>(off[E]) * f;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / f), n = static_cast<int>(i - static_cast<long long>(m) * f);
    const int e = expert_of_row(off, E, m);
    const float* xr = x + static_cast<size_t>(m) * d;
    const size_t wrow = (static_cast<size_t>(e) * f + n) * d;
    const float gsum = dot_f32(xr, wg + wrow, d);
    const float usum = dot_f32(xr, wu + wrow, d);
    h[i] = gsum / (1.f + expf(-gsum)) * usum;
  }
}

__global__ void down_f32_kernel(const float* __restrict__ h, const int32_t* __restrict__ offsets, int E, int d, int f,
                                const float* __restrict__ wd, float* __restrict__ y) {
  __shared__ int off[65];
  if (threadIdx.x <= E) off[threadIdx.x] = offsets[threadIdx.x];
  __syncthreads();
  const long long total = static_cast<long long>(off[E]) * d;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(i / d), n = static_cast<int>(i - static_cast<long long>(m) * d);
    const int e = expert_of_row(off, E, m);
    y[i] = dot_f32(h + static_cast<size_t>(m) * f, wd + (static_cast<size_t>(e) * d + n) * f, f);
  }
}

// Average rows per expert at or above which the tensor-core GEMM path is used.
constexpr int kTcMinRowsPerExpert = 64;

}  // namespace
}  // namespace zmoe

extern "C" {

size_t zmoe_grouped_swiglu_workspace_size(int M_total, int E, int d, int f, zmoe_dtype dtype) {
  if (M_total < 0 || E < 1 || d < 1 || f < 1) return 0;
  if (dtype == ZMOE_BF16) {
    const size_t a = zmoe::grouped_swiglu_tc_workspace(M_total, E, d, f);
    const size_t b = zmoe::grouped_swiglu_dec_tc_workspace(M_total, E, d, f);
    return a > b ? a : b;
  }
  return 0;
}

zmoe_status zmoe_grouped_swiglu(const void* x_perm, const int32_t* offsets, int M_total, const void* w_gate,
                                const void* w_up, const void* w_down, zmoe_dtype dtype, int E, int d, int f, void* h,
                                float* y_perm, void* workspace, size_t ws_bytes, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_grouped_swiglu");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_grouped_swiglu: bad dtype");
  ZMOE_REQUIRE(M_total >= 0, "zmoe_grouped_swiglu: M_total must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_grouped_swiglu: E must be in [1, 64]");
  ZMOE_REQUIRE(d >= 8 && f >= 8, "zmoe_grouped_swiglu: d and f must be >= 8");
  ZMOE_REQUIRE(offsets != nullptr, "zmoe_grouped_swiglu: offsets is NULL");
  if (M_total == 0) return ZMOE_OK;
  ZMOE_REQUIRE(x_perm && w_gate && w_up && w_down && h && y_perm, "zmoe_grouped_swiglu: NULL pointer");
  ZMOE_REQUIRE(aligned16(x_perm) && aligned16(w_gate) && aligned16(w_up) && aligned16(w_down) && aligned16(h) &&
                   aligned16(y_perm),
               "zmoe_grouped_swiglu: pointers must be 16-byte aligned");
  ZMOE_REQUIRE(static_cast<long long>(M_total) * (d > f ? d : f) <= 0x7fffffffLL,
               "zmoe_grouped_swiglu: M_total * max(d, f) overflows int32");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == ZMOE_F32) {
    ZMOE_REQUIRE(d % 4 == 0 && f % 4 == 0, "zmoe_grouped_swiglu: f32 needs d % 4 == 0 and f % 4 == 0");
    long long grid = (static_cast<long long>(M_total) * (d > f ? d : f) + 255) / 256;
    const long long cap = static_cast<long long>(num_sms()) * 8;
    if (grid > cap) grid = cap;
    gateup_f32_kernel<<<static_cast<int>(grid), 256, 0, s>>>(static_cast<const float*>(x_perm), offsets, E, d, f,
                                                             static_cast<const float*>(w_gate),
                                                             static_cast<const float*>(w_up), static_cast<float*>(h));
    down_f32_kernel<<<static_cast<int>(grid), 256, 0, s>>>(static_cast<const float*>(h), offsets, E, d, f,
                                                           static_cast<const float*>(w_down), y_perm);
    return check_launch("zmoe_grouped_swiglu (f32)");
  }
  ZMOE_REQUIRE(d % 256 == 0 && f % 256 == 0, "zmoe_grouped_swiglu: bf16 needs d % 256 == 0 and f % 256 == 0");
  const auto* xp = static_cast<const uint16_t*>(x_perm);
  const auto* wg = static_cast<const uint16_t*>(w_gate);
  const auto* wu = static_cast<const uint16_t*>(w_up);
  const auto* wd = static_cast<const uint16_t*>(w_down);
  auto* hh = static_cast<uint16_t*>(h);
  const bool tc_ok = grouped_swiglu_tc_supported(d, f);
  const bool dec_ok = grouped_swiglu_dec_tc_supported(d, f);
  if (tc_ok && (M_total >= kTcMinRowsPerExpert * E || !dec_ok)) {
    if (ws_bytes < grouped_swiglu_tc_workspace(M_total, E, d, f))
      return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                  "zmoe_grouped_swiglu: workspace smaller than zmoe_grouped_swiglu_workspace_size()");
    return grouped_swiglu_tc(xp, offsets, M_total, wg, wu, wd, E, d, f, hh, y_perm, workspace, ws_bytes, s);
  }
  if (!dec_ok) return fail(ZMOE_ERR_UNSUPPORTED, "zmoe_grouped_swiglu: no bf16 kernel for this d, f");
  if (!workspace || ws_bytes < grouped_swiglu_dec_tc_workspace(M_total, E, d, f))
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                "zmoe_grouped_swiglu: workspace smaller than zmoe_grouped_swiglu_workspace_size()");
  return grouped_swiglu_dec_tc(xp, offsets, M_total, wg, wu, wd, E, d, f, hh, y_perm, workspace, s);
}

zmoe_status zmoe_grouped_swiglu_f16h(const void* x_perm, const int32_t* offsets, int M_total, const void* w_gate,
                                     const void* w_up, const void* w_down_f16, const float* down_scale, int E, int d,
                                     int f, void* h, float* y_perm, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_grouped_swiglu_f16h");
  using namespace zmoe;
  ZMOE_REQUIRE(M_total >= 0, "zmoe_grouped_swiglu_f16h: M_total must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_grouped_swiglu_f16h: E must be in [1, 64]");
  ZMOE_REQUIRE(d >= 256 && f >= 256 && d % 256 == 0 && f % 256 == 0,
               "zmoe_grouped_swiglu_f16h: d and f must be multiples of 256");
  ZMOE_REQUIRE(offsets != nullptr, "zmoe_grouped_swiglu_f16h: offsets is NULL");
  if (M_total == 0) return ZMOE_OK;
  ZMOE_REQUIRE(x_perm && w_gate && w_up && w_down_f16 && down_scale && h && y_perm,
               "zmoe_grouped_swiglu_f16h: NULL pointer");
  ZMOE_REQUIRE(aligned16(x_perm) && aligned16(w_gate) && aligned16(w_up) && aligned16(w_down_f16) && aligned16(h) &&
                   aligned16(y_perm),
               "zmoe_grouped_swiglu_f16h: pointers must be 16-byte aligned");
  ZMOE_REQUIRE(static_cast<long long>(M_total) * (d > f ? d : f) <= 0x7fffffffLL,
               "zmoe_grouped_swiglu_f16h: M_total * max(d, f) overflows int32");
  clear_error();
  return grouped_swiglu_tc_f16h(static_cast<const uint16_t*>(x_perm), offsets, M_total,
                                static_cast<const uint16_t*>(w_gate), static_cast<const uint16_t*>(w_up),
                                static_cast<const uint16_t*>(w_down_f16), down_scale, E, d, f, static_cast<uint16_t*>(h),
                                y_perm, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"
