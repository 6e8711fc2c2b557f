// Delay pattern over the RVQ codebooks (ZONOS2 Technical Report digest, "method overview
// and architecture", item 1): Y[t, j] = X[t - j, j] and its inverse X_hat[t, j] = Y[t + j, j].
//
// Pure index work: one thread per output element, consecutive threads write consecutive
// int32 words of the output (coalesced); reads are strided by N - 1 words per codebook
// column, which stays within the same few cache lines for N = 9.
#include "common.cuh"

namespace zmoe {
namespace {

__global__ void shear_kernel(const int32_t* __restrict__ X, int32_t* __restrict__ Y, int B, int T, int N,
                             int32_t pad) {
  const int Ty = T + N - 1;
  const long long total = static_cast<long long>(B) * Ty * N;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i % N);
    const long long bt = i / N;
    const int t = static_cast<int>(bt % Ty);
    const long long b = bt / Ty;
    const int src = t - j;
    Y[i] = (src >= 0 && src < T) ? X[(b * T + src) * N + j] : pad;
  }
}

__global__ void unshear_kernel(const int32_t* __restrict__ Y, int32_t* __restrict__ X, int B, int Ty, int N) {
  const int T = Ty - N + 1;
  const long long total = static_cast<long long>(B) * T * N;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int j = static_cast<int>(i % N);
    const long long bt = i / N;
    const int t = static_cast<int>(bt % T);
    const long long b = bt / T;
    X[i] = Y[(b * Ty + t + j) * N + j];
  }
}

int grid_for(long long total, int block) {
  long long g = (total + block - 1) / block;
  const long long cap = static_cast<long long>(num_sms()) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace
}  // namespace zmoe

extern "C" {

zmoe_status zmoe_delay_shear(const int32_t* X, int32_t* Y, int B, int T, int N, int32_t pad,
                             zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_delay_shear");
  using namespace zmoe;
  ZMOE_REQUIRE(B >= 0 && T >= 0, "zmoe_delay_shear: B and T must be >= 0");
  ZMOE_REQUIRE(N >= 1 && N <= 64, "zmoe_delay_shear: N must be in [1, 64]");
  const long long total = static_cast<long long>(B) * (T + N - 1) * N;
  if (B == 0) return ZMOE_OK;
  ZMOE_REQUIRE(Y != nullptr, "zmoe_delay_shear: Y is NULL");
  ZMOE_REQUIRE(T == 0 || X != nullptr, "zmoe_delay_shear: X is NULL");
  clear_error();
  shear_kernel<<<grid_for(total, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(X, Y, B, T, N, pad);
  return check_launch("zmoe_delay_shear");
}

zmoe_status zmoe_delay_unshear(const int32_t* Y, int32_t* X, int B, int Ty, int N, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_delay_unshear");
  using namespace zmoe;
  ZMOE_REQUIRE(B >= 0, "zmoe_delay_unshear: B must be >= 0");
  ZMOE_REQUIRE(N >= 1 && N <= 64, "zmoe_delay_unshear: N must be in [1, 64]");
  ZMOE_REQUIRE(Ty >= N - 1, "zmoe_delay_unshear: Ty must be >= N - 1");
  const long long total = static_cast<long long>(B) * (Ty - N + 1) * N;
  if (total == 0) return ZMOE_OK;
  ZMOE_REQUIRE(X != nullptr && Y != nullptr, "zmoe_delay_unshear: NULL pointer");
  clear_error();
  unshear_kernel<<<grid_for(total, 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(Y, X, B, Ty, N);
  return check_launch("zmoe_delay_unshear");
}

}  // extern "C"
