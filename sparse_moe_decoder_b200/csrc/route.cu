// Router: logits, selection-only bias, top-k, softmax gates.
//
// ZONOS2 Technical Report digest, "method overview and architecture", items 5-6 (16 experts,
// top-1 routing, top-2 in the last MoE layer; a per-layer bias b_l steers expert usage), the
// telknet.cc article on ZONOS2, section 2.1 (linear router followed by TopK), and
// "Auxiliary-Loss-Free Load Balancing" (ZONOS2 Technical Report, "Builds on"): the bias moves
// the selection, not the gate values.
//   q = W_r x + logit_bias;  s = q + sel_bias;  top-k of s (ties -> lower index);
//   p = softmax(q);  k = 1: gate = p[sel];  k = 2: gates renormalised over the two.
//
// Work split: a CTA of 8 warps owns TB = 64 / EP tokens (EP = E padded to 16, 32 or 64).  The
// d-range is cut into 256-wide chunks dealt round-robin to the 8 warps; lane l of a warp owns
// the 8 consecutive elements [c*256 + 8l, c*256 + 8l + 8) of chunk c.  Each lane accumulates all
// TB x EP partial logits (64 fp32 registers), a reduce-scatter butterfly over the warp leaves
// lane l with the two complete partial sums of entries 2l and 2l + 1 (token 2l / EP, experts
// (2l) % EP and +1), the 8 warps' partials are summed through shared memory, and top-k and the
// softmax run inside the EP/2-lane group that holds one token.  x is read once from HBM with
// 16-byte loads; W_r is read through the read-only cache (it is shared by all CTAs).
#include <math.h>

#include "common.cuh"

namespace zmoe {

bool launch_route_tc(const void* x, const void* w, const float* lb, const float* sb, int T, int d, int E, int k,
                     int32_t* idx, float* g, float* mg, cudaStream_t s);

namespace {

constexpr int kWarps = 8;

template <typename T>
__device__ __forceinline__ void load8v(const T* p, float* v);

template <>
__device__ __forceinline__ void load8v<uint16_t>(const uint16_t* p, float* v) {
  unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(p)), v);
}

template <>
__device__ __forceinline__ void load8v<float>(const float* p, float* v) {
  float4 a = __ldg(reinterpret_cast<const float4*>(p));
  float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

// Candidate order: larger score first, then lower expert index.
__device__ __forceinline__ bool better(float s, int e, float s2, int e2) {
  return s > s2 || (s == s2 && e < e2);
}

// Best (score, index) over a group of G lanes (G a power of two, groups aligned).
template <int G>
__device__ __forceinline__ void group_argmax(float& s, int& e) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) {
    float so = __shfl_xor_sync(0xffffffffu, s, o);
    int eo = __shfl_xor_sync(0xffffffffu, e, o);
    if (better(so, eo, s, e)) {
      s = so;
      e = eo;
    }
  }
}

template <int G>
__device__ __forceinline__ float group_max(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <int G>
__device__ __forceinline__ float group_sum(float v) {
#pragma unroll
  for (int o = G / 2; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Top-k, gates and margin of one token from the logits its G = EP / 2 lanes hold: lane l of the group
// holds the (unbiased) logits l0, l1 of experts 2 (l % G) and 2 (l % G) + 1.  Lane 0 of the group writes.
template <int EP>
__device__ __forceinline__ void finish_topk(float l0, float l1, int tok, int lane, int T_, int E, int k,
                                            const float* __restrict__ logit_bias, const float* __restrict__ sel_bias,
                                            int32_t* __restrict__ expert_idx, float* __restrict__ gates,
                                            float* __restrict__ margin) {
  constexpr int G = EP / 2;
  const int ea = (2 * lane) % EP, eb = ea + 1;
  const bool va = ea < E, vb = eb < E;
  const float NEG = -INFINITY;
  float qa = va ? l0 + (logit_bias ? logit_bias[ea] : 0.f) : NEG;
  float qb = vb ? l1 + (logit_bias ? logit_bias[eb] : 0.f) : NEG;
  float sa = va ? qa + (sel_bias ? sel_bias[ea] : 0.f) : NEG;
  float sb = vb ? qb + (sel_bias ? sel_bias[eb] : 0.f) : NEG;

  // rank 1
  float s1 = sa;
  int e1 = va ? ea : 0x7fffffff;
  if (vb && better(sb, eb, s1, e1)) {
    s1 = sb;
    e1 = eb;
  }
  group_argmax<G>(s1, e1);
  // rank 2: best candidate other than e1
  float s2 = NEG;
  int e2 = 0x7fffffff;
  if (va && ea != e1) {
    s2 = sa;
    e2 = ea;
  }
  if (vb && eb != e1 && better(sb, eb, s2, e2)) {
    s2 = sb;
    e2 = eb;
  }
  group_argmax<G>(s2, e2);
  // rank 3 (margin of top-2 only)
  float s3 = NEG;
  if (k == 2) {
    int e3 = 0x7fffffff;
    if (va && ea != e1 && ea != e2) {
      s3 = sa;
      e3 = ea;
    }
    if (vb && eb != e1 && eb != e2 && better(sb, eb, s3, e3)) {
      s3 = sb;
      e3 = eb;
    }
    group_argmax<G>(s3, e3);
  }

  // softmax over the unbiased q of this token
  const float m = group_max<G>(fmaxf(qa, qb));
  const float za = va ? expf(qa - m) : 0.f;
  const float zb = vb ? expf(qb - m) : 0.f;
  const float zsum = group_sum<G>(za + zb);
  // fetch q of the selected experts from the lanes that hold them
  const int gbase = (lane / G) * G;
  const float q1 = __shfl_sync(0xffffffffu, (e1 & 1) ? qb : qa, gbase + ((e1 % EP) >> 1));
  float q2 = NEG;
  if (k == 2) q2 = __shfl_sync(0xffffffffu, (e2 & 1) ? qb : qa, gbase + ((e2 % EP) >> 1));

  if ((lane % G) == 0 && tok < T_) {
    if (k == 1) {
      expert_idx[tok] = e1;
      gates[tok] = expf(q1 - m) / zsum;
      if (margin) margin[tok] = (E > 1) ? s1 - s2 : INFINITY;
    } else {
      const float z1 = expf(q1 - m), z2 = expf(q2 - m);
      const float inv = 1.f / (z1 + z2);
      expert_idx[2 * tok] = e1;
      expert_idx[2 * tok + 1] = e2;
      gates[2 * tok] = z1 * inv;
      gates[2 * tok + 1] = z2 * inv;
      if (margin) margin[tok] = (E > 2) ? fminf(s1 - s2, s2 - s3) : s1 - s2;
    }
  }
}

template <typename T, int EP>
__global__ void __launch_bounds__(kWarps * 32) route_kernel(
    const T* __restrict__ x, const T* __restrict__ w, const float* __restrict__ logit_bias,
    const float* __restrict__ sel_bias, int T_, int d, int E, int k, int32_t* __restrict__ expert_idx,
    float* __restrict__ gates, float* __restrict__ margin) {
  constexpr int TB = 64 / EP;   // tokens per CTA (EP / 2 lanes hold one token's logits)
  __shared__ float2 part[kWarps][32];

  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int t0 = blockIdx.x * TB;

  float acc[TB * EP];
#pragma unroll
  for (int i = 0; i < TB * EP; ++i) acc[i] = 0.f;

  for (int c = warp; c * 256 < d; c += kWarps) {
    const int k0 = c * 256 + lane * 8;
    if (k0 < d) {
      float xv[TB][8];
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) {
        if (t0 + tb < T_) {
          load8v<T>(x + static_cast<size_t>(t0 + tb) * d + k0, xv[tb]);
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) xv[tb][i] = 0.f;
        }
      }
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E) {
          float wv[8];
          load8v<T>(w + static_cast<size_t>(e) * d + k0, wv);
#pragma unroll
          for (int tb = 0; tb < TB; ++tb) {
#pragma unroll
            for (int i = 0; i < 8; ++i) acc[tb * EP + e] = fmaf(wv[i], xv[tb][i], acc[tb * EP + e]);
          }
        }
      }
    }
  }

  // Reduce-scatter over the warp: after the step with offset o, a lane keeps the upper half
  // of its current values when (lane & o) != 0.  After 5 steps lane l holds entries 2l, 2l+1.
#pragma unroll
  for (int o = 16, n = 64; o > 0; o >>= 1, n >>= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float send = upper ? acc[i] : acc[i + n / 2];
      const float keep = upper ? acc[i + n / 2] : acc[i];
      acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
    }
  }
  part[warp][lane] = make_float2(acc[0], acc[1]);
  __syncthreads();
  if (warp != 0) return;

  float l0 = 0.f, l1 = 0.f;
#pragma unroll
  for (int w2 = 0; w2 < kWarps; ++w2) {
    l0 += part[w2][lane].x;
    l1 += part[w2][lane].y;
  }
  finish_topk<EP>(l0, l1, t0 + (2 * lane) / EP, lane, T_, E, k, logit_bias, sel_bias, expert_idx, gates, margin);
}

// Prefill sizes (bf16, E <= 16): persistent CTAs stage the whole router matrix in shared memory once;
// each warp takes TB = 4 tokens at a time over the whole d (lane l: elements [c 256 + 8 l, + 8) of every
// chunk c), so no partial sums cross warps and each router byte read from memory serves every token of
// the CTA.  The per-token sums then take the same reduce-scatter and top-k as route_kernel.
template <int EP>
__global__ void __launch_bounds__(kWarps * 32) route_rows_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ w, const float* __restrict__ logit_bias,
    const float* __restrict__ sel_bias, int T_, int d, int E, int k, int32_t* __restrict__ expert_idx,
    float* __restrict__ gates, float* __restrict__ margin) {
  constexpr int TB = 64 / EP;
  extern __shared__ uint4 wsm[];   // [E][d / 8] 16-byte vectors of bf16
  const int vecs = E * (d / 8);
  for (int i = threadIdx.x; i < vecs; i += blockDim.x) wsm[i] = __ldg(reinterpret_cast<const uint4*>(w) + i);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int groups = (T_ + TB - 1) / TB;
  const int dv = d / 8;
  for (int gi = blockIdx.x * kWarps + warp; gi < groups; gi += gridDim.x * kWarps) {
    const int t0 = gi * TB;
    float acc[TB * EP];
#pragma unroll
    for (int i = 0; i < TB * EP; ++i) acc[i] = 0.f;
    // x chunks are loaded one chunk ahead of the arithmetic (the raw 16-byte vectors stay packed)
    uint4 xn[TB];
    const int nch = (d + 255) / 256;
    auto load_chunk = [&](int c, uint4 (&dst)[TB]) {
      const int k0 = c * 256 + lane * 8;
#pragma unroll
      for (int tb = 0; tb < TB; ++tb)
        dst[tb] = (k0 < d && t0 + tb < T_) ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t0 + tb) * d + k0))
                                           : make_uint4(0u, 0u, 0u, 0u);
    };
    load_chunk(0, xn);
    for (int c = 0; c < nch; ++c) {
      const int k0 = c * 256 + lane * 8;
      float xv[TB][8];
#pragma unroll
      for (int tb = 0; tb < TB; ++tb) unpack_bf16x8(xn[tb], xv[tb]);
      if (c + 1 < nch) load_chunk(c + 1, xn);
      if (k0 < d) {
#pragma unroll
        for (int e = 0; e < EP; ++e) {
          if (e < E) {
            float wv[8];
            unpack_bf16x8(wsm[e * dv + (k0 >> 3)], wv);
#pragma unroll
            for (int tb = 0; tb < TB; ++tb) {
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[tb * EP + e] = fmaf(wv[i], xv[tb][i], acc[tb * EP + e]);
            }
          }
        }
      }
    }
#pragma unroll
    for (int o = 16, n = 64; o > 0; o >>= 1, n >>= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < n / 2; ++i) {
        const float send = upper ? acc[i] : acc[i + n / 2];
        const float keep = upper ? acc[i + n / 2] : acc[i];
        acc[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
      }
    }
    finish_topk<EP>(acc[0], acc[1], t0 + (2 * lane) / EP, lane, T_, E, k, logit_bias, sel_bias, expert_idx, gates,
                    margin);
  }
}

// Tokens from which the persistent CUDA-core router kernel is used (below, the one-CTA-per-4-tokens kernel needs no
// staging of the router matrix).
constexpr int kRowsMinT = 512;

template <typename T>
void launch_route(const void* x, const void* w, const float* lb, const float* sb, int T_, int d, int E, int k,
                  int32_t* idx, float* g, float* mg, cudaStream_t s) {
  const T* xp = static_cast<const T*>(x);
  const T* wp = static_cast<const T*>(w);
  const size_t wbytes = static_cast<size_t>(E) * d * sizeof(T);
  // the tensor-core router (bf16, E <= 32, d % 64 == 0, T >= 2048)
  if (sizeof(T) == 2 && launch_route_tc(x, w, lb, sb, T_, d, E, k, idx, g, mg, s)) return;
  if (sizeof(T) == 2 && E <= 16 && T_ >= kRowsMinT && wbytes <= 96 * 1024) {
    auto kern = route_rows_kernel<16>;
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(wbytes)) ==
        cudaSuccess) {
      const int groups = (T_ + 3) / 4;
      int grid = 2 * num_sms();   // two CTAs per SM (128 registers, <= 96 KB each), persistent over the groups
      if (grid * kWarps > groups) grid = (groups + kWarps - 1) / kWarps;
      kern<<<grid, kWarps * 32, wbytes, s>>>(reinterpret_cast<const uint16_t*>(xp), reinterpret_cast<const uint16_t*>(wp),
                                              lb, sb, T_, d, E, k, idx, g, mg);
      return;
    }
    cudaGetLastError();
  }
  if (E <= 16) {
    route_kernel<T, 16><<<(T_ + 3) / 4, kWarps * 32, 0, s>>>(xp, wp, lb, sb, T_, d, E, k, idx, g, mg);
  } else if (E <= 32) {
    route_kernel<T, 32><<<(T_ + 1) / 2, kWarps * 32, 0, s>>>(xp, wp, lb, sb, T_, d, E, k, idx, g, mg);
  } else {
    route_kernel<T, 64><<<T_, kWarps * 32, 0, s>>>(xp, wp, lb, sb, T_, d, E, k, idx, g, mg);
  }
}

// E == 1 without a router: expert 0, gate softmax over one logit = 1, no second choice (margin +inf).
__global__ void single_expert_kernel(int T, int32_t* __restrict__ expert_idx, float* __restrict__ gates,
                                     float* __restrict__ margin) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < T) {
    expert_idx[t] = 0;
    gates[t] = 1.f;
    if (margin) margin[t] = INFINITY;
  }
}

}  // namespace
}  // namespace zmoe

extern "C" zmoe_status zmoe_route(const void* x, const void* w_router, zmoe_dtype dtype, const float* logit_bias,
                                  const float* sel_bias, int T, int d, int E, int k, int32_t* expert_idx,
                                  float* gates, float* margin, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_route");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_route: bad dtype");
  ZMOE_REQUIRE(T >= 0, "zmoe_route: T must be >= 0");
  ZMOE_REQUIRE(E >= 1 && E <= 64, "zmoe_route: E must be in [1, 64]");
  ZMOE_REQUIRE(k == 1 || k == 2, "zmoe_route: k must be 1 or 2");
  ZMOE_REQUIRE(k <= E, "zmoe_route: k must be <= E");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0, "zmoe_route: d must be a positive multiple of 8");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE(expert_idx && gates && (!w_router ? E == 1 : x != nullptr),
               "zmoe_route: NULL pointer (w_router may be NULL only when E == 1)");
  ZMOE_REQUIRE((!x || aligned16(x)) && (!w_router || aligned16(w_router)), "zmoe_route: x/w_router not 16-byte aligned");
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (!w_router) {
    // one expert and no router (a dense FFN layer): every token goes to expert 0 with gate 1
    single_expert_kernel<<<(T + 255) / 256, 256, 0, s>>>(T, expert_idx, gates, margin);
    return check_launch("zmoe_route");
  }
  if (dtype == ZMOE_BF16)
    launch_route<uint16_t>(x, w_router, logit_bias, sel_bias, T, d, E, k, expert_idx, gates, margin, s);
  else
    launch_route<float>(x, w_router, logit_bias, sel_bias, T, d, E, k, expert_idx, gates, margin, s);
  return check_launch("zmoe_route");
}
