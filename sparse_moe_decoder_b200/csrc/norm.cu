// Summed codebook embeddings + RMSNorm, and plain row RMSNorm.
//
// ZONOS2 Technical Report digest, "method overview and architecture", item 5: the decoder
// input is the sum of the embeddings of the (delayed) codebook frame, normalised by RMSNorm
// ("Root Mean Square Layer Normalization", listed under "Builds on" of the ZONOS2 Technical
// Report).  out = e / sqrt(mean(e^2) + eps) * gamma, with e accumulated in fp32.
//
// One CTA per row.  Each thread owns 8-element vectors (16-byte loads of bf16, two 16-byte
// loads of f32), keeps e in shared memory in fp32, and the CTA reduces sum(e^2) with warp
// shuffles.  HBM-bound: the row's N table rows are read once and the output written once.
#include "common.cuh"

namespace zmoe {
namespace {

constexpr int kThreads = 256;

template <typename T>
__device__ __forceinline__ void load8(const T* p, float* v);

template <>
__device__ __forceinline__ void load8<uint16_t>(const uint16_t* p, float* v) {
  uint4 raw = *reinterpret_cast<const uint4*>(p);
  unpack_bf16x8(raw, v);
}

template <>
__device__ __forceinline__ void load8<float>(const float* p, float* v) {
  float4 a = reinterpret_cast<const float4*>(p)[0];
  float4 b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

template <typename T>
__device__ __forceinline__ void store8(T* p, const float* v);

template <>
__device__ __forceinline__ void store8<uint16_t>(uint16_t* p, const float* v) {
  uint4 o;
  o.x = pack_bf16x2(v[0], v[1]);
  o.y = pack_bf16x2(v[2], v[3]);
  o.z = pack_bf16x2(v[4], v[5]);
  o.w = pack_bf16x2(v[6], v[7]);
  *reinterpret_cast<uint4*>(p) = o;
}

template <>
__device__ __forceinline__ void store8<float>(float* p, const float* v) {
  reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
  reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Sum over the CTA; every thread receives the total.
__device__ __forceinline__ float block_sum(float v, float* scratch) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  float t = (lane < (kThreads / 32)) ? scratch[lane] : 0.f;
  t = warp_sum(t);
  return t;
}

// Normalises the fp32 row held in `e_smem` and writes it out.
template <typename TOut>
__device__ __forceinline__ void normalise_store(const float* e_smem, float sumsq, const float* __restrict__ gamma,
                                                float eps, int d, TOut* __restrict__ out_row) {
  const float inv = rsqrtf(sumsq / static_cast<float>(d) + eps);
  for (int v = threadIdx.x; v < d / 8; v += kThreads) {
    float x[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = e_smem[v * 8 + i] * inv * __ldg(gamma + v * 8 + i);
    store8<TOut>(out_row + static_cast<size_t>(v) * 8, x);
  }
}

template <typename TTab, typename TOut>
__global__ void __launch_bounds__(kThreads) embed_sum_rmsnorm_kernel(
    const int32_t* __restrict__ ids, const TTab* __restrict__ tables, const float* __restrict__ gamma, float eps,
    int N, int V, int d, TOut* __restrict__ out, unsigned int* err) {
  extern __shared__ float e_smem[];
  __shared__ float red[kThreads / 32];
  __shared__ int row_ids[64];
  const int t = blockIdx.x;
  if (threadIdx.x < N) {
    int id = ids[static_cast<size_t>(t) * N + threadIdx.x];
    if (id < 0 || id >= V) {
      record_device_error(err);
      id = -1;
    }
    row_ids[threadIdx.x] = id;
  }
  __syncthreads();
  float sumsq = 0.f;
  for (int v = threadIdx.x; v < d / 8; v += kThreads) {
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j < N; ++j) {
      const int id = row_ids[j];
      if (id < 0) continue;
      float x[8];
      load8<TTab>(tables + (static_cast<size_t>(j) * V + id) * d + static_cast<size_t>(v) * 8, x);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] += x[i];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      e_smem[v * 8 + i] = acc[i];
      sumsq += acc[i] * acc[i];
    }
  }
  sumsq = block_sum(sumsq, red);
  normalise_store<TOut>(e_smem, sumsq, gamma, eps, d, out + static_cast<size_t>(t) * d);
}

template <typename TIn, typename TOut>
__global__ void __launch_bounds__(kThreads) rmsnorm_kernel(const TIn* __restrict__ h, const float* __restrict__ gamma,
                                                           float eps, int d, TOut* __restrict__ out) {
  extern __shared__ float e_smem[];
  __shared__ float red[kThreads / 32];
  const int t = blockIdx.x;
  float sumsq = 0.f;
  for (int v = threadIdx.x; v < d / 8; v += kThreads) {
    float x[8];
    load8<TIn>(h + static_cast<size_t>(t) * d + static_cast<size_t>(v) * 8, x);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      e_smem[v * 8 + i] = x[i];
      sumsq += x[i] * x[i];
    }
  }
  sumsq = block_sum(sumsq, red);
  normalise_store<TOut>(e_smem, sumsq, gamma, eps, d, out + static_cast<size_t>(t) * d);
}

template <typename K>
zmoe_status set_smem(K kernel, size_t bytes, const char* what) {
  if (bytes > 48 * 1024) {
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
        cudaSuccess)
      return check_launch(what);
  }
  return ZMOE_OK;
}

}  // namespace
}  // namespace zmoe

extern "C" {

zmoe_status zmoe_embed_sum_rmsnorm(const int32_t* ids, const void* tables, zmoe_dtype table_dtype,
                                   const float* gamma, float eps, int T, int N, int V, int d, void* out,
                                   zmoe_dtype out_dtype, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_embed_sum_rmsnorm");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(table_dtype) && dtype_ok(out_dtype), "zmoe_embed_sum_rmsnorm: bad dtype");
  ZMOE_REQUIRE(T >= 0 && N >= 1 && N <= 64 && V >= 1, "zmoe_embed_sum_rmsnorm: bad T, N or V");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0, "zmoe_embed_sum_rmsnorm: d must be a positive multiple of 8");
  ZMOE_REQUIRE(eps >= 0.f, "zmoe_embed_sum_rmsnorm: eps must be >= 0");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE(ids && tables && gamma && out, "zmoe_embed_sum_rmsnorm: NULL pointer");
  ZMOE_REQUIRE(aligned16(tables) && aligned16(out), "zmoe_embed_sum_rmsnorm: tables/out not 16-byte aligned");
  const size_t smem = static_cast<size_t>(d) * sizeof(float);
  ZMOE_REQUIRE(smem <= static_cast<size_t>(max_smem_optin()), "zmoe_embed_sum_rmsnorm: d too large");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int* err = device_error_counter();
  zmoe_status st = ZMOE_OK;
#define ZMOE_EMBED_LAUNCH(TT, TO)                                                                           \
  do {                                                                                                      \
    auto k = embed_sum_rmsnorm_kernel<TT, TO>;                                                              \
    if ((st = set_smem(k, smem, "zmoe_embed_sum_rmsnorm")) != ZMOE_OK) return st;                           \
    k<<<T, kThreads, smem, s>>>(ids, static_cast<const TT*>(tables), gamma, eps, N, V, d, static_cast<TO*>(out), \
                                err);                                                                       \
  } while (0)
  if (table_dtype == ZMOE_BF16 && out_dtype == ZMOE_BF16) ZMOE_EMBED_LAUNCH(uint16_t, uint16_t);
  else if (table_dtype == ZMOE_BF16) ZMOE_EMBED_LAUNCH(uint16_t, float);
  else if (out_dtype == ZMOE_BF16) ZMOE_EMBED_LAUNCH(float, uint16_t);
  else ZMOE_EMBED_LAUNCH(float, float);
#undef ZMOE_EMBED_LAUNCH
  return check_launch("zmoe_embed_sum_rmsnorm");
}

zmoe_status zmoe_rmsnorm(const void* h, zmoe_dtype in_dtype, const float* gamma, float eps, int T, int d, void* out,
                         zmoe_dtype out_dtype, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_rmsnorm");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(in_dtype) && dtype_ok(out_dtype), "zmoe_rmsnorm: bad dtype");
  ZMOE_REQUIRE(T >= 0, "zmoe_rmsnorm: T must be >= 0");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0, "zmoe_rmsnorm: d must be a positive multiple of 8");
  ZMOE_REQUIRE(eps >= 0.f, "zmoe_rmsnorm: eps must be >= 0");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE(h && gamma && out, "zmoe_rmsnorm: NULL pointer");
  ZMOE_REQUIRE(aligned16(h) && aligned16(out), "zmoe_rmsnorm: h/out not 16-byte aligned");
  const size_t smem = static_cast<size_t>(d) * sizeof(float);
  ZMOE_REQUIRE(smem <= static_cast<size_t>(max_smem_optin()), "zmoe_rmsnorm: d too large");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  zmoe_status st = ZMOE_OK;
#define ZMOE_NORM_LAUNCH(TI, TO)                                                                         \
  do {                                                                                                   \
    auto k = rmsnorm_kernel<TI, TO>;                                                                     \
    if ((st = set_smem(k, smem, "zmoe_rmsnorm")) != ZMOE_OK) return st;                                 \
    k<<<T, kThreads, smem, s>>>(static_cast<const TI*>(h), gamma, eps, d, static_cast<TO*>(out));         \
  } while (0)
  if (in_dtype == ZMOE_BF16 && out_dtype == ZMOE_BF16) ZMOE_NORM_LAUNCH(uint16_t, uint16_t);
  else if (in_dtype == ZMOE_BF16) ZMOE_NORM_LAUNCH(uint16_t, float);
  else if (out_dtype == ZMOE_BF16) ZMOE_NORM_LAUNCH(float, uint16_t);
  else ZMOE_NORM_LAUNCH(float, float);
#undef ZMOE_NORM_LAUNCH
  return check_launch("zmoe_rmsnorm");
}

}  // extern "C"
