// zmoe_output_heads: the 9 codebook heads on the final hidden state and the greedy next frame.
//
// ZONOS2 Technical Report digest, "method overview and architecture", items 1 and 5: the decoder
// predicts the next frame Y[t+1, n] of the 9 delay-patterned DAC codebooks.  Per token t:
//   x = RMSNorm(h[t]) * gamma (optional final norm), rounded to bf16 like every layer input;
//   logits[t, n, v] = sum_c W_heads[n, v, c] x[c]      (fp32 accumulation, one bias-free head per codebook)
//   ids[t, n] = argmax_v logits[t, n, v]               (ties -> the lower id)
//
// At decode sizes the work is streaming the heads' N V d weights (37.8 MB in bf16) from HBM once per
// 8 tokens.  One CTA per SM takes an equal contiguous range of the N V head rows, streams it through
// a shared-memory ring with TMA bulk copies (rows are contiguous), and each warp dots one row with the
// 8 staged token rows.  The argmax is a 64-bit atomicMax on (order-preserving logit bits, ~v) per
// (token, codebook): order-independent, so the result does not depend on which CTA finishes first;
// the last CTA to finish decodes the ids.
#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int kThreads = 256;     // 8 warps
constexpr int kWarps = kThreads / 32;
constexpr int kRowsPerStage = kWarps;   // one head row per warp per stage
constexpr int kTok = 8;           // tokens per pass over the weights
constexpr int kMaxStages = 8;
constexpr int kXC = 8;            // a single bf16 token row of d <= 256 kXC is held in registers
constexpr unsigned long long kTimeoutNs = 2000000000ull;

struct HeadArgs {
  const float* h;            // [T, d]
  const float* gamma;        // [d] or null
  float eps;
  const unsigned char* w;    // [N * V, d] of elem bytes
  int elem;                  // 2 (bf16) or 4 (f32)
  int T, N, V, d;
  int stages;                // ring depth
  int32_t* ids;              // [T, N]
  float* logits;             // [T, N, V] or null
  uint16_t* x_out;           // [T, d] bf16 or null (the routed input as rounded)
  unsigned long long* keys;  // [T, N] zeroed before the launch
  unsigned int* done;        // CTAs finished, zeroed before the launch
  unsigned int* timeouts;
  unsigned int* errors;
};

struct __align__(8) HeadCtrl {
  uint64_t full[kMaxStages];
  uint64_t empty[kMaxStages];   // every warp is done with the slot (one arrival per warp)
  uint64_t xbar;             // token rows (+ gamma) of the current pass
  unsigned long long best[kWarps][kTok][2];   // each warp's best key per token for the CTA's two codebooks
  float red[kWarps][kTok];   // per-warp partial sums of squares (the final norm)
  int abort;
};

constexpr size_t kCtrlBytes = 1536;
static_assert(sizeof(HeadCtrl) <= kCtrlBytes, "the control block must fit ahead of the token rows");

// Dynamic shared memory: control | token rows f32 [kTok][d] (x is formed in place, rounded to the weights'
// type but kept as f32) | gamma f32 [d] | weight ring.
struct HeadSmem {
  size_t raw, gam, ring, total;
};

__host__ __device__ inline size_t a128(size_t b) { return (b + 127) & ~static_cast<size_t>(127); }

// tok = token rows per pass (min(T, kTok)): a batch-1 call leaves the room to the weight ring.
__host__ __device__ inline HeadSmem head_smem(int d, int elem, int stages, int tok) {
  HeadSmem S;
  S.raw = kCtrlBytes;
  S.gam = S.raw + a128(static_cast<size_t>(tok) * d * 4);
  S.ring = S.gam + a128(static_cast<size_t>(d) * 4);
  S.total = S.ring + static_cast<size_t>(stages) * d * elem * kRowsPerStage;
  return S;
}

// Order-preserving map of a float onto uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t ordered_bits(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Columns [c, c + 8) of one head row against the pass's token rows x (f32 in shared memory).
__device__ __forceinline__ void dot8(const unsigned char* wrow, int elem, int c, const float* xs, int d, int nt,
                                     float (&acc)[kTok]) {
  float w8[8];
  if (elem == 2) {
    unpack_bf16x8(*reinterpret_cast<const uint4*>(wrow + static_cast<size_t>(c) * 2), w8);
  } else {
    const float4 a = *reinterpret_cast<const float4*>(wrow + static_cast<size_t>(c) * 4);
    const float4 b = *reinterpret_cast<const float4*>(wrow + static_cast<size_t>(c) * 4 + 16);
    w8[0] = a.x; w8[1] = a.y; w8[2] = a.z; w8[3] = a.w;
    w8[4] = b.x; w8[5] = b.y; w8[6] = b.z; w8[7] = b.w;
  }
#pragma unroll
  for (int t = 0; t < kTok; ++t) {
    if (t < nt) {
      const float4 p = *reinterpret_cast<const float4*>(xs + static_cast<size_t>(t) * d + c);
      const float4 q = *reinterpret_cast<const float4*>(xs + static_cast<size_t>(t) * d + c + 4);
      acc[t] = fmaf(w8[0], p.x, acc[t]);
      acc[t] = fmaf(w8[1], p.y, acc[t]);
      acc[t] = fmaf(w8[2], p.z, acc[t]);
      acc[t] = fmaf(w8[3], p.w, acc[t]);
      acc[t] = fmaf(w8[4], q.x, acc[t]);
      acc[t] = fmaf(w8[5], q.y, acc[t]);
      acc[t] = fmaf(w8[6], q.z, acc[t]);
      acc[t] = fmaf(w8[7], q.w, acc[t]);
    }
  }
}

// Issues ring stage `s` (rows [r0 + 8 s, ...)) into `slot` (thread 0).
__device__ __forceinline__ void issue_stage(const HeadArgs& a, HeadCtrl& C, unsigned char* ring, size_t slot_bytes,
                                           int slot, int r0, int r1, int s) {
  const size_t row_bytes = static_cast<size_t>(a.d) * a.elem;
  const int rs = r0 + s * kRowsPerStage;
  const int nrows = (r1 - rs) < kRowsPerStage ? (r1 - rs) : kRowsPerStage;
  const uint32_t bytes = static_cast<uint32_t>(nrows * row_bytes);
  unsigned char* dst = ring + static_cast<size_t>(slot) * slot_bytes;
  const unsigned char* src = a.w + static_cast<size_t>(rs) * row_bytes;
  mbar_expect_tx(&C.full[slot], bytes);
  for (uint32_t o = 0; o < bytes; o += 32768u) {
    const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
    bulk_load(dst + o, src + o, n, &C.full[slot]);
  }
}

__global__ void __launch_bounds__(kThreads, 1) heads_kernel(HeadArgs a) {
  extern __shared__ __align__(128) unsigned char smem[];
  HeadCtrl& C = *reinterpret_cast<HeadCtrl*>(smem);
  const int d = a.d, N = a.N, V = a.V;
  const HeadSmem L = head_smem(d, a.elem, a.stages, a.T < kTok ? a.T : kTok);
  float* raw = reinterpret_cast<float*>(smem + L.raw);
  float* gam = reinterpret_cast<float*>(smem + L.gam);
  float* xs = raw;   // x is formed in place
  unsigned char* ring = smem + L.ring;
  const size_t row_bytes = static_cast<size_t>(d) * a.elem;
  const size_t slot_bytes = row_bytes * kRowsPerStage;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long R = static_cast<long long>(N) * V;
  const int r0 = static_cast<int>(R * blockIdx.x / gridDim.x), r1 = static_cast<int>(R * (blockIdx.x + 1) / gridDim.x);
  const int nst = (r1 - r0 + kRowsPerStage - 1) / kRowsPerStage;
  volatile int* abort_flag = &C.abort;
  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], kWarps);
    }
    mbar_init(&C.xbar, 1);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const int n0 = r0 / V;   // a CTA's rows touch codebooks n0 and (at most) n0 + 1: rows per CTA < V
  int q = 0;   // stages issued over all passes (slot = q % stages, parity = (q / stages) & 1)
  bool ok = true;
  for (int t0 = 0; t0 < a.T && ok; t0 += kTok) {
    const int nt = (a.T - t0) < kTok ? (a.T - t0) : kTok;
    // the pass's token rows (and gamma, first pass) by bulk copy, one round trip, then its first weight
    // stages, which do not depend on x and land while x is formed
    const int pass = t0 / kTok;
    if (threadIdx.x == 0) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      const uint32_t rb = static_cast<uint32_t>(nt) * d * 4u;
      const uint32_t gb = (pass == 0 && a.gamma) ? static_cast<uint32_t>(d) * 4u : 0u;
      mbar_expect_tx(&C.xbar, rb + gb);
      for (uint32_t o = 0; o < rb; o += 32768u)
        bulk_load(reinterpret_cast<unsigned char*>(raw) + o,
                  reinterpret_cast<const unsigned char*>(a.h + static_cast<size_t>(t0) * d) + o,
                  rb - o < 32768u ? rb - o : 32768u, &C.xbar);
      for (uint32_t o = 0; o < gb; o += 32768u)
        bulk_load(reinterpret_cast<unsigned char*>(gam) + o, reinterpret_cast<const unsigned char*>(a.gamma) + o,
                  gb - o < 32768u ? gb - o : 32768u, &C.xbar);
      for (int s = 0; s < nst && s < a.stages; ++s) issue_stage(a, C, ring, slot_bytes, (q + s) % a.stages, r0, r1, s);
    }
    ok = __syncthreads_and(mbar_wait(&C.xbar, static_cast<uint32_t>(pass & 1), abort_flag, kTimeoutNs));
    if (!ok) {
      if (threadIdx.x == 0) {
        if (atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
        const uint64_t t1 = globaltimer();
        while (!mbar_try_wait(&C.xbar, static_cast<uint32_t>(pass & 1)) && globaltimer() - t1 < kTimeoutNs) {
        }
        // the weight stages issued above must land before the CTA leaves
        for (int s2 = 0; s2 < nst && s2 < a.stages; ++s2) {
          const int slot = (q + s2) % a.stages;
          const uint32_t par = static_cast<uint32_t>(((q + s2) / a.stages) & 1);
          const uint64_t t2 = globaltimer();
          while (!mbar_try_wait(&C.full[slot], par) && globaltimer() - t2 < kTimeoutNs) {
          }
        }
      }
      break;
    }
    // optional RMSNorm of each token row, by the whole CTA (sums of squares per thread, then per warp,
    // then over the warps), and rounding to the weights' type
    float inv[kTok];
#pragma unroll
    for (int t = 0; t < kTok; ++t) inv[t] = 1.f;
    if (a.gamma) {
      float ss[kTok];
#pragma unroll
      for (int t = 0; t < kTok; ++t) ss[t] = 0.f;
      for (int c = threadIdx.x; c < d; c += kThreads) {
#pragma unroll
        for (int t = 0; t < kTok; ++t)
          if (t < nt) ss[t] = fmaf(raw[static_cast<size_t>(t) * d + c], raw[static_cast<size_t>(t) * d + c], ss[t]);
      }
#pragma unroll
      for (int t = 0; t < kTok; ++t) {
        if (t < nt) {
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) ss[t] += __shfl_xor_sync(0xffffffffu, ss[t], o);
          if (lane == 0) C.red[warp][t] = ss[t];
        }
      }
      __syncthreads();
#pragma unroll
      for (int t = 0; t < kTok; ++t) {
        if (t < nt) {
          float tot = 0.f;
#pragma unroll
          for (int w = 0; w < kWarps; ++w) tot += C.red[w][t];
          inv[t] = rsqrtf(tot / static_cast<float>(d) + a.eps);
        }
      }
    }
    for (int c = threadIdx.x; c < d; c += kThreads) {
#pragma unroll
      for (int t = 0; t < kTok; ++t) {
        if (t >= nt) continue;
        const size_t i = static_cast<size_t>(t) * d + c;
        const float v = a.gamma ? raw[i] * inv[t] * gam[c] : raw[i];
        // in place over raw (element i was read above by this thread only)
        if (a.elem == 2) {
          const uint16_t b = f32_to_bf16_bits(v);
          xs[i] = bf16_to_f32(b);
          if (a.x_out && blockIdx.x == 0) a.x_out[static_cast<size_t>(t0) * d + i] = b;
        } else {
          xs[i] = v;
          if (a.x_out && blockIdx.x == 0) reinterpret_cast<float*>(a.x_out)[static_cast<size_t>(t0) * d + i] = v;
        }
      }
    }
    __syncthreads();
    // one bf16 token: its row in registers (lane's 8-column chunks), the weights alone from shared memory
    const bool x1 = nt == 1 && a.elem == 2 && d <= 256 * kXC;
    float xr[kXC][8];
#pragma unroll
    for (int j = 0; j < kXC; ++j) {
      const int c = lane * 8 + j * 256;
      if (x1 && c < d) {
        const float4 p = *reinterpret_cast<const float4*>(xs + c);
        const float4 q = *reinterpret_cast<const float4*>(xs + c + 4);
        xr[j][0] = p.x; xr[j][1] = p.y; xr[j][2] = p.z; xr[j][3] = p.w;
        xr[j][4] = q.x; xr[j][5] = q.y; xr[j][6] = q.z; xr[j][7] = q.w;
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) xr[j][i] = 0.f;
      }
    }
    // lane t < nt of every warp keeps the warp's best key of token t for codebooks n0 and n0 + 1
    unsigned long long best0 = 0ull, best1 = 0ull;
    int issued = nst < a.stages ? nst : a.stages;   // thread 0: stages of this pass issued so far
    int s = 0;
    for (; s < nst; ++s) {
      const int slot = (q + s) % a.stages;
      const uint32_t par = static_cast<uint32_t>(((q + s) / a.stages) & 1);
      ok = __all_sync(0xffffffffu, mbar_wait(&C.full[slot], par, abort_flag, kTimeoutNs));
      if (!ok) {   // stop the other warps' waits too
        if (lane == 0 && atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
        break;
      }
      const int rs = r0 + s * kRowsPerStage;
      if (rs + warp < r1) {
        const unsigned char* wrow = ring + static_cast<size_t>(slot) * slot_bytes + static_cast<size_t>(warp) * row_bytes;
        float acc[kTok];
#pragma unroll
        for (int t = 0; t < kTok; ++t) acc[t] = 0.f;
        if (x1) {   // four partial sums (chunks j mod 4), added pairwise: short dependency chains
          float p4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int j = 0; j < kXC; ++j) {
            const int c = lane * 8 + j * 256;
            if (c < d) {
              float w8[8];
              unpack_bf16x8(*reinterpret_cast<const uint4*>(wrow + static_cast<size_t>(c) * 2), w8);
#pragma unroll
              for (int i = 0; i < 8; ++i) p4[j & 3] = fmaf(w8[i], xr[j][i], p4[j & 3]);
            }
          }
          acc[0] = (p4[0] + p4[1]) + (p4[2] + p4[3]);
        } else {
          for (int c = lane * 8; c < d; c += 256) dot8(wrow, a.elem, c, xs, d, nt, acc);
        }
#pragma unroll
        for (int t = 0; t < kTok; ++t) {
          if (t < nt) {   // warp-uniform
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], o);
          }
        }
        // every lane holds every sum: lane t takes token t's
        float lg = acc[0];
#pragma unroll
        for (int t = 1; t < kTok; ++t)
          if (lane == t) lg = acc[t];
        const int row = rs + warp;
        const int n = row / V, v = row - n * V;
        if (lane < nt) {
          if (a.logits) a.logits[(static_cast<size_t>(t0 + lane) * N + n) * V + v] = lg;
          if (lg == lg) {   // NaN never wins
            const unsigned long long key = (static_cast<unsigned long long>(ordered_bits(lg)) << 32) |
                                           static_cast<unsigned long long>(0xFFFFFFFFu - static_cast<uint32_t>(v));
            if (n == n0) best0 = key > best0 ? key : best0;
            else best1 = key > best1 ? key : best1;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[slot]);
      // thread 0 refills the slot once every warp is done with it
      if (threadIdx.x == 0 && s + a.stages < nst) {
        if (!mbar_wait(&C.empty[slot], par, abort_flag, kTimeoutNs)) {
          ok = false;
          if (atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
        } else {
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          issue_stage(a, C, ring, slot_bytes, slot, r0, r1, s + a.stages);
          ++issued;
        }
      }
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
    }
    ok = __syncthreads_and(ok && !*abort_flag);
    if (!ok) {
      if (threadIdx.x == 0) {
        if (atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
        // copies issued but not consumed must land before the CTA leaves: the last stage issued into
        // each slot (the slot's latest phase)
        for (int s2 = issued > a.stages ? issued - a.stages : 0; s2 < issued; ++s2) {
          const int slot = (q + s2) % a.stages;
          const uint32_t par = static_cast<uint32_t>(((q + s2) / a.stages) & 1);
          const uint64_t t1 = globaltimer();
          while (!mbar_try_wait(&C.full[slot], par) && globaltimer() - t1 < kTimeoutNs) {
          }
        }
      }
      break;
    }
    // the CTA's best key per (token, codebook) over its warps, then one global atomic each:
    // order-independent, so deterministic
    if (lane < kTok) {
      C.best[warp][lane][0] = best0;
      C.best[warp][lane][1] = best1;
    }
    __syncthreads();
    if (threadIdx.x < 2 * nt) {
      const int t = threadIdx.x >> 1, j = threadIdx.x & 1;
      unsigned long long key = 0ull;
#pragma unroll
      for (int w = 0; w < kWarps; ++w) key = C.best[w][t][j] > key ? C.best[w][t][j] : key;
      if (key != 0ull && n0 + j < N) atomicMax(a.keys + static_cast<size_t>(t0 + t) * N + n0 + j, key);
    }
    __syncthreads();   // C.best is rewritten by the next pass
    q += nst;
  }
  // the last CTA to finish turns the keys into ids
  __shared__ int last;
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    last = atomicAdd(a.done, 1u) == gridDim.x - 1;
    __threadfence();
  }
  __syncthreads();
  if (last) {
    for (int i = threadIdx.x; i < a.T * N; i += kThreads) {
      const unsigned long long key = __ldcg(a.keys + i);
      if (key == 0ull) {
        a.ids[i] = -1;   // every logit of this (token, codebook) was NaN
        record_device_error(a.errors);
      } else {
        a.ids[i] = static_cast<int32_t>(0xFFFFFFFFu - static_cast<uint32_t>(key & 0xFFFFFFFFull));
      }
    }
  }
}

}  // namespace
}  // namespace zmoe

extern "C" {

size_t zmoe_output_heads_workspace_size(int T, int N) {
  if (T < 0 || N < 1) return 0;
  return ((static_cast<size_t>(T) * N * 8 + 16) + 255) & ~static_cast<size_t>(255);
}

zmoe_status zmoe_output_heads(const float* h, const float* gamma, float eps, const void* w_heads, zmoe_dtype dtype,
                              int T, int N, int V, int d, int32_t* ids, float* logits, void* x_out, void* workspace,
                              size_t ws_bytes, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_output_heads");
  using namespace zmoe;
  ZMOE_REQUIRE(dtype_ok(dtype), "zmoe_output_heads: bad dtype");
  ZMOE_REQUIRE(T >= 0 && N >= 1 && V >= 1, "zmoe_output_heads: T >= 0, N >= 1, V >= 1");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0, "zmoe_output_heads: d must be a positive multiple of 8");
  ZMOE_REQUIRE(static_cast<long long>(N) * V <= 0x7fffffffLL, "zmoe_output_heads: N * V overflows int32");
  ZMOE_REQUIRE(eps >= 0.f, "zmoe_output_heads: eps must be >= 0");
  if (T == 0) return ZMOE_OK;
  ZMOE_REQUIRE(h && w_heads && ids, "zmoe_output_heads: NULL pointer");
  ZMOE_REQUIRE(aligned16(w_heads) && aligned16(h) && (!gamma || aligned16(gamma)),
               "zmoe_output_heads: h, gamma and w_heads must be 16-byte aligned");
  if (!workspace || ws_bytes < zmoe_output_heads_workspace_size(T, N))
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                "zmoe_output_heads: workspace smaller than zmoe_output_heads_workspace_size()");
  const int elem = static_cast<int>(dtype_size(dtype));
  const size_t slot_bytes = static_cast<size_t>(d) * elem * kRowsPerStage;
  const size_t budget = static_cast<size_t>(max_smem_optin()) - 1024;   // room for the static shared word
  const int tok = T < kTok ? T : kTok;
  const size_t fixed = head_smem(d, elem, 0, tok).total;
  if (budget < fixed + 2 * slot_bytes)
    return fail(ZMOE_ERR_UNSUPPORTED, "zmoe_output_heads: d too large for the shared-memory ring");
  int stages = static_cast<int>((budget - fixed) / slot_bytes);
  if (stages > kMaxStages) stages = kMaxStages;
  const size_t smem = head_smem(d, elem, stages, tok).total;
  clear_error();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const size_t key_bytes = static_cast<size_t>(T) * N * 8;
  if (cudaMemsetAsync(workspace, 0, key_bytes + 16, s) != cudaSuccess) return check_launch("zmoe_output_heads: memset");
  if (cudaFuncSetAttribute(heads_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return check_launch("zmoe_output_heads: shared memory attribute");
  HeadArgs a{};
  a.h = h;
  a.gamma = gamma;
  a.eps = eps;
  a.w = static_cast<const unsigned char*>(w_heads);
  a.elem = elem;
  a.T = T;
  a.N = N;
  a.V = V;
  a.d = d;
  a.stages = stages;
  a.ids = ids;
  a.logits = logits;
  a.x_out = static_cast<uint16_t*>(x_out);
  a.keys = static_cast<unsigned long long*>(workspace);
  a.done = reinterpret_cast<unsigned int*>(static_cast<unsigned char*>(workspace) + key_bytes);
  a.timeouts = device_timeout_counter();
  a.errors = device_error_counter();
  const long long rows = static_cast<long long>(N) * V;
  // at least N CTAs, so that a CTA's contiguous rows span at most two codebooks
  long long grid_l = num_sms();
  if (grid_l < N) grid_l = N;
  if (rows < grid_l) grid_l = rows;
  const int grid = static_cast<int>(grid_l);
  heads_kernel<<<grid, kThreads, smem, s>>>(a);
  return check_launch("zmoe_output_heads");
}

}  // extern "C"
