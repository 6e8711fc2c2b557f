// Gate-weighted combine: y[t] = sum_i gates[t, i] * y_perm[inv_perm[t, i]] (+ residual[t]).
//
// The telknet.cc article on ZONOS2, section 2.1: the layer output is the gate-weighted sum of
// the top-k experts' outputs.  Written as a per-token GATHER in fixed slot order (slot 0, then
// slot 1, then the residual), so the result is deterministic and needs no atomics; it is the
// same sum a scatter-add would form.  HBM-bound: one 16-byte load per slot and one 16-byte
// store per 4 outputs.  `y` may alias `residual` (each element is read before it is written by
// the same thread), so neither is declared __restrict__.
#include "common.cuh"

namespace zmoe {
namespace {

__global__ void combine_kernel(const float4* __restrict__ y_perm, const int32_t* __restrict__ inv_perm,
                               const float* __restrict__ gates, const float4* residual, int T, int vecs, int k,
                               float4* y, unsigned int* err) {
  const long long total = static_cast<long long>(T) * vecs;
  const int rows = T * k;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / vecs);
    const int v = static_cast<int>(i - static_cast<long long>(t) * vecs);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < k; ++s) {
      const int r = __ldg(inv_perm + t * k + s);
      if (r < 0 || r >= rows) {
        if (v == 0) record_device_error(err);
        continue;
      }
      const float g = __ldg(gates + t * k + s);
      const float4 yp = __ldg(y_perm + static_cast<size_t>(r) * vecs + v);
      acc.x = fmaf(g, yp.x, acc.x);
      acc.y = fmaf(g, yp.y, acc.y);
      acc.z = fmaf(g, yp.z, acc.z);
      acc.w = fmaf(g, yp.w, acc.w);
    }
    if (residual) {
      const float4 rv = residual[i];
      acc.x += rv.x;
      acc.y += rv.y;
      acc.z += rv.z;
      acc.w += rv.w;
    }
    y[i] = acc;
  }
}

}  // namespace
}  // namespace zmoe

extern "C" zmoe_status zmoe_combine(const float* y_perm, const int32_t* inv_perm, const float* gates,
                                    const float* residual, int T, int d, int k, float* y, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_combine");
  using namespace zmoe;
  ZMOE_REQUIRE(T >= 0, "zmoe_combine: T must be >= 0");
  ZMOE_REQUIRE(k == 1 || k == 2, "zmoe_combine: k must be 1 or 2");
  ZMOE_REQUIRE(d >= 4 && d % 4 == 0, "zmoe_combine: d must be a positive multiple of 4");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE(y_perm && inv_perm && gates && y, "zmoe_combine: NULL pointer");
  ZMOE_REQUIRE(aligned16(y_perm) && aligned16(y) && (!residual || aligned16(residual)),
               "zmoe_combine: y_perm/y/residual not 16-byte aligned");
  ZMOE_REQUIRE(static_cast<long long>(T) * k <= 0x7fffffffLL, "zmoe_combine: T * k overflows int32");
  clear_error();
  const int vecs = d / 4;
  const long long total = static_cast<long long>(T) * vecs;
  long long grid = (total + 255) / 256;
  const long long cap = static_cast<long long>(num_sms()) * 8;
  if (grid > cap) grid = cap;
  combine_kernel<<<static_cast<int>(grid), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      reinterpret_cast<const float4*>(y_perm), inv_perm, gates, reinterpret_cast<const float4*>(residual), T, vecs, k,
      reinterpret_cast<float4*>(y), device_error_counter());
  return check_launch("zmoe_combine");
}
