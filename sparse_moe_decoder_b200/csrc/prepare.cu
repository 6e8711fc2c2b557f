// One-time preparation of the down-projection weights for the f16 hidden-activation prefill path.
//
// The tensor cores take both operands of one MMA in the same 16-bit format.  The prefill down GEMM
// carries h in f16 (11 significant bits, enough for the bf16 bar; a single bf16 h is not), so W_down
// must be f16 too.  bf16 has 8 significant bits and an 8-bit exponent, f16 has 11 bits and a 5-bit
// exponent: a bf16 value converts to f16 exactly when it lies in f16's normal range.  Each expert's
// weights are therefore scaled by a power of two 2^s_e that moves its largest magnitude into
// [2^14, 2^15) before the conversion:
//   w16[e] = f16(w_down[e] * 2^s_e)   (exact for every |w| >= 2^(e_max - 28), e_max = exponent of the
//                                      largest |w| of the expert; smaller values round to f16's
//                                      subnormals with an absolute error of at most 2^(e_max - 39))
//   down_scale[e] = 2^-s_e            (the down GEMM multiplies its fp32 sums by it: exact)
// Three launches: the largest magnitude per expert (fp32 bits compared as integers), the conversion,
// and the scales.  Deterministic; the result does not depend on the launch order of CTAs.
#include "common.cuh"

namespace zmoe {
namespace {

constexpr int kThreads = 256;

// Largest |w| of each expert, as the bit pattern of a non-negative float (ordered like the values).
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint4* __restrict__ w, long long vecs_per_expert,
                                                         unsigned int* __restrict__ amax_bits) {
  const int e = blockIdx.y;
  const uint4* we = w + static_cast<size_t>(e) * vecs_per_expert;
  unsigned int m = 0;
  for (long long i = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; i < vecs_per_expert;
       i += static_cast<long long>(gridDim.x) * kThreads) {
    const uint4 v = we[i];
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // |bf16| as fp32 bits: clear the sign, widen
      const unsigned int lo = (words[j] & 0x7FFFu) << 16, hi = (words[j] >> 16 & 0x7FFFu) << 16;
      m = max(m, max(lo, hi));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits + e, m);
}

// The exponent shift s_e for an expert whose largest magnitude has these fp32 bits.
__device__ __forceinline__ int shift_of(unsigned int amax_bits) {
  if (amax_bits == 0u || amax_bits >= 0x7F800000u) return 0;   // all zero (or non-finite: left unscaled)
  int ex;
  frexpf(__uint_as_float(amax_bits), &ex);                      // amax = m 2^ex, m in [0.5, 1)
  const int s = 15 - ex;                                        // amax 2^s in [2^14, 2^15)
  return s < -100 ? -100 : (s > 100 ? 100 : s);
}

__global__ void __launch_bounds__(kThreads) convert_kernel(const uint4* __restrict__ w, long long vecs_per_expert,
                                                            int E, const unsigned int* __restrict__ amax_bits,
                                                            uint4* __restrict__ w16) {
  const long long total = vecs_per_expert * E;
  for (long long i = blockIdx.x * static_cast<long long>(kThreads) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * kThreads) {
    const int e = static_cast<int>(i / vecs_per_expert);
    const float sc = ldexpf(1.f, shift_of(amax_bits[e]));
    const uint4 v = w[i];
    const uint32_t words[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float a = __uint_as_float(words[j] << 16) * sc, b = __uint_as_float(words[j] & 0xFFFF0000u) * sc;
      const __half ha = __float2half_rn(a), hb = __float2half_rn(b);
      out[j] = static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&ha)) |
               (static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&hb)) << 16);
    }
    w16[i] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

__global__ void scale_kernel(const unsigned int* __restrict__ amax_bits, int E, float* __restrict__ down_scale) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e < E) down_scale[e] = ldexpf(1.f, -shift_of(amax_bits[e]));
}

}  // namespace
}  // namespace zmoe

extern "C" zmoe_status zmoe_prepare_w_down_f16(const void* w_down, int E, int d, int f, void* w_down_f16,
                                               float* down_scale, void* workspace, size_t ws_bytes,
                                               zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_prepare_w_down_f16");
  using namespace zmoe;
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_prepare_w_down_f16: E must be in [1, 64]");
  ZMOE_REQUIRE(d >= 8 && f >= 8 && d % 8 == 0 && f % 8 == 0, "zmoe_prepare_w_down_f16: d, f must be multiples of 8");
  ZMOE_REQUIRE(w_down && w_down_f16 && down_scale, "zmoe_prepare_w_down_f16: NULL pointer");
  ZMOE_REQUIRE(aligned16(w_down) && aligned16(w_down_f16), "zmoe_prepare_w_down_f16: pointers must be 16-byte aligned");
  if (!workspace || ws_bytes < static_cast<size_t>(E) * 4)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL, "zmoe_prepare_w_down_f16: workspace needs 4 E bytes");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* amax = static_cast<unsigned int*>(workspace);
  const long long vpe = static_cast<long long>(d) * f / 8;   // 16-byte vectors per expert
  if (cudaMemsetAsync(amax, 0, static_cast<size_t>(E) * 4, s) != cudaSuccess)
    return check_launch("zmoe_prepare_w_down_f16: clearing");
  const int per = static_cast<int>((vpe + kThreads * 8 - 1) / (kThreads * 8));
  amax_kernel<<<dim3(static_cast<unsigned>(per < 64 ? per : 64), static_cast<unsigned>(E)), kThreads, 0, s>>>(
      static_cast<const uint4*>(w_down), vpe, amax);
  const long long cap = static_cast<long long>(num_sms()) * 8;
  long long grid = (vpe * E + kThreads - 1) / kThreads;
  if (grid > cap) grid = cap;
  convert_kernel<<<static_cast<int>(grid), kThreads, 0, s>>>(static_cast<const uint4*>(w_down), vpe, E, amax,
                                                              static_cast<uint4*>(w_down_f16));
  scale_kernel<<<1, 64, 0, s>>>(amax, E, down_scale);
  return check_launch("zmoe_prepare_w_down_f16");
}
