// zmoe_speaker_prefix: the speaker-embedding row prepended to the decoder input.
//
// ZONOS2 Technical Report digest, "method overview and architecture", item 3: the ECAPA-TDNN
// speaker embedding, reduced by LDA to 1024 values e, is projected to the model width,
//   h_spk[b] = W_spk e[b] + b_spk            (fp32 accumulation)
// and placed at position 0 of the input sequence.  A small GEMV (d x 1024 weights, 4 MB in bf16):
// one warp per output row, each lane with all of its 16-byte weight loads in flight before it
// multiplies, the embeddings staged once per CTA in shared memory.
#include "common.cuh"

namespace zmoe {
namespace {

constexpr int kThreads = 256;   // 8 warps = 8 output rows per CTA
constexpr int kWarps = kThreads / 32;
constexpr int kB = 8;           // embeddings per pass

template <typename TW>
__device__ __forceinline__ void load8w(const TW* p, float* v);

template <>
__device__ __forceinline__ void load8w<uint16_t>(const uint16_t* p, float* v) {
  unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(p)), v);
}

template <>
__device__ __forceinline__ void load8w<float>(const float* p, float* v) {
  const float4 a = __ldg(reinterpret_cast<const float4*>(p)), b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename TW>
__global__ void __launch_bounds__(kThreads) speaker_kernel(const float* __restrict__ e, const TW* __restrict__ w,
                                                           const float* __restrict__ bias, int B, int d, int n_in,
                                                           float* __restrict__ out) {
  extern __shared__ float es[];   // [kB][n_in]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * kWarps + warp;
  for (int b0 = 0; b0 < B; b0 += kB) {
    const int nb = (B - b0) < kB ? (B - b0) : kB;
    __syncthreads();   // the previous pass is done with es
    for (int i = threadIdx.x; i < nb * n_in; i += kThreads) es[i] = __ldg(e + static_cast<size_t>(b0) * n_in + i);
    __syncthreads();
    if (row >= d) continue;
    const TW* wr = w + static_cast<size_t>(row) * n_in;
    float acc[kB];
#pragma unroll
    for (int j = 0; j < kB; ++j) acc[j] = 0.f;
    for (int c0 = lane * 8; c0 < n_in; c0 += 4 * 256) {
      float wv[4][8];
#pragma unroll
      for (int u = 0; u < 4; ++u)   // four loads in flight before any multiply
        if (c0 + u * 256 < n_in) load8w<TW>(wr + c0 + u * 256, wv[u]);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int c = c0 + u * 256;
        if (c < n_in) {
#pragma unroll
          for (int j = 0; j < kB; ++j)
            if (j < nb) {
              const float* er = es + j * n_in + c;
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[j] = fmaf(wv[u][i], er[i], acc[j]);
            }
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kB; ++j) {
      if (j < nb) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
        if (lane == 0) out[static_cast<size_t>(b0 + j) * d + row] = acc[j] + (bias ? bias[row] : 0.f);
      }
    }
  }
}

}  // namespace
}  // namespace zmoe

extern "C" zmoe_status zmoe_speaker_prefix(const float* e, const void* w_spk, zmoe_dtype dtype, const float* b_spk,
                                           int B, int d, int n_in, float* out, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_speaker_prefix");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_speaker_prefix: bad dtype");
  ZMOE_REQUIRE(B >= 0 && d >= 1 && n_in >= 8 && n_in % 8 == 0, "zmoe_speaker_prefix: B >= 0, d >= 1, n_in % 8 == 0");
  if (B == 0) return ZMOE_OK;
  ZMOE_REQUIRE(e && w_spk && out, "zmoe_speaker_prefix: NULL pointer");
  ZMOE_REQUIRE(aligned16(w_spk), "zmoe_speaker_prefix: w_spk must be 16-byte aligned");
  const size_t smem = static_cast<size_t>(kB) * n_in * 4;
  ZMOE_REQUIRE(smem <= 200 * 1024, "zmoe_speaker_prefix: n_in too large");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int grid = (d + kWarps - 1) / kWarps;
  if (dtype == ZMOE_BF16) {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(speaker_kernel<uint16_t>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return check_launch("zmoe_speaker_prefix");
    speaker_kernel<uint16_t><<<grid, kThreads, smem, s>>>(e, static_cast<const uint16_t*>(w_spk), b_spk, B, d, n_in,
                                                          out);
  } else {
    if (smem > 48 * 1024 &&
        cudaFuncSetAttribute(speaker_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(smem)) != cudaSuccess)
      return check_launch("zmoe_speaker_prefix");
    speaker_kernel<float><<<grid, kThreads, smem, s>>>(e, static_cast<const float*>(w_spk), b_spk, B, d, n_in, out);
  }
  return check_launch("zmoe_speaker_prefix");
}
