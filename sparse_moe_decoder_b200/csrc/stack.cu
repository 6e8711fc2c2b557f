// The batch-1 decode stack in ONE persistent cooperative launch: the summed codebook embeddings +
// RMSNorm (optional), then every layer's pre-norm residual block
//   x = bf16(RMSNorm(h) * gamma_l),  h <- h + sum_i gate_i * W_down[e_i] (silu(W_gate[e_i] x) * (W_up[e_i] x))
// with the router (logits + selection bias, top-k, softmax gates) of each layer, or gate 1 for a dense
// FFN layer (E = 1, no router).  ZONOS2 digest, "method overview and architecture", item 5 (the decoder
// input is the RMSNorm of the summed embeddings of the 9 codebooks; 3 dense FFN layers, 24 MoE layers of
// 16 experts, top-1 and top-2 in the last MoE layer, 1 dense layer); the telknet.cc article on ZONOS2,
// section 2.1 (router, gate-weighted sum of the chosen experts).  The pre-norm residual wiring is the
// reading taken for the block.
//
// One token: every layer is two matrix-vector passes over the chosen experts' weights (37.75 MB per
// expert at d = 2048, f = 3072), so the step is bound by HBM and by the latency between layers.  A
// launch per layer pays the launch, the staging of the router rows and the first weight bytes every
// time; here one launch runs all layers and per layer only two grid barriers separate the phases:
//   * every CTA repeats the pre-norm, the router logits and the selection (no barrier before the
//     weights); the router rows and gain of layer l + 1 are bulk-copied into shared memory at the end of
//     layer l (while its grid barrier runs), so routing starts from shared memory;
//   * phase A: CTA c owns the f-rows [c f / C, (c + 1) f / C) of each chosen expert.  These rows are
//     contiguous in W_gate and W_up, so one producer thread streams them as blocks of up to 7 rows,
//     one bulk copy per ring slot (~28 KB: one SM's streaming rate grows with the copy size, 4 KB copies
//     reach well under half of it); gate and up blocks alternate, 7 consumer warps take every slot in
//     order, warp w row w of the block (the gate value waits in shared memory for the up row); h goes
//     to global memory in fp32;
//   * grid barrier 1 (consumers only: the producer keeps streaming W_down blocks), a bulk copy of h
//     into the router rows' area;
//   * phase B: CTA c owns the d-rows [c d / C, (c + 1) d / C) (blocks of up to 5 rows of W_down, ~30 KB),
//     contracts them and adds the chosen experts, in slot order, to its rows of the residual stream h
//     (in global memory, in place);
//   * grid barrier 2 (all of h updated) before the next layer's pre-norm.
// Every sum is fp32 in a fixed order (no atomics on data): results do not depend on timing.  Every
// wait is bounded; on expiry the CTA counts a timeout, stops, waits (bounded) for its own copies in
// flight and returns.
#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int kThreads = 256;            // warp 0: producer; warps 1..7: consumers
constexpr int kConsumers = 7;
constexpr int kSlots = 4;                // every consumer warp takes every slot, in order
constexpr uint32_t kSlotTarget = 32768;  // bytes of weights per slot (at most)
constexpr int kMaxK = 2;
constexpr int kMaxE = 64;
constexpr int kMaxLayers = 32;
constexpr int kMaxRowsB = 64;            // d-rows per CTA
constexpr int kMaxVec = 2;               // 8-element vectors of the residual stream per thread
constexpr int kMaxN = 32;                // codebooks
constexpr unsigned long long kTimeoutNs = 2000000000ull;

struct StackLayerDev {
  const uint16_t* w_r;       // [E, d] or null (E == 1: gate 1)
  const float* logit_bias;   // [E] or null
  const float* sel_bias;     // [E] or null
  const float* gamma;        // [d]
  const uint16_t* w_gate;    // [E, f, d]
  const uint16_t* w_up;      // [E, f, d]
  const uint16_t* w_down;    // [E, d, f]
  int E, k;
};

struct StackArgs {
  StackLayerDev L[kMaxLayers];
  int n_layers, d, f, N, V;
  float eps;
  const int32_t* ids;        // [N] or null: then h holds the stack input on entry
  const uint16_t* tables;    // [N, V, d]
  const float* gamma0;       // [d]
  float* h;                  // [d] residual stream, in place
  float* hbuf;               // [kMaxK, f] h of the current layer
  unsigned int* gbar;        // grid barrier arrivals (zeroed before the launch)
  unsigned int* timeouts;
  unsigned int* errors;
  int32_t* layer_idx;        // [n_layers, 2] or null (-1 past k)
  float* layer_gates;        // [n_layers, 2] or null (0 past k)
  float* layer_h;            // [n_layers, d] or null: h entering each layer
  uint16_t* layer_x;         // [n_layers, d] or null: each layer's input as routed (bf16)
  uint32_t slot_bytes;       // max(ra 2 d, rb 2 f), a multiple of 128
  uint32_t r1_bytes;         // max(E d 2 over layers, kMaxK f 4), a multiple of 16
  int ra, rb;                // rows per phase-A block (<= 7) and per phase-B block (<= 7)
};

struct __align__(16) StackCtrl {
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t st;               // staging of a layer's router rows and gain: one phase per layer
  uint64_t hb;               // the layer's h, after grid barrier 1: one phase per layer
  uint64_t r1free;           // phase B has read h: the area may take the next router rows (one per layer)
  int abort;
  int nu;                    // chosen experts (= k): slot i holds expert uexp[i] with gate gsel[i]
  int uexp[kMaxK];
  float gsel[kMaxK];
  int ids[kMaxN];
  float red[kThreads / 32];
  float lpart[kThreads / 32][kMaxE];   // per-warp partial router logits
  float qb[kMaxE];           // the layer's logit bias (0 when none)
  float sb[kMaxE];           // the layer's selection bias (0 when none)
  float gv[kConsumers];      // gate value of warp w's row of the current block
  float ypart[kMaxK][kMaxRowsB];
};

// Shared memory: ring | R1 (router rows, then h of the chosen experts in phase B) | gamma | x (f32) |
// control.
struct StackSmem {
  size_t ring, r1, gam, xs, ctrl, total;
};

__host__ __device__ inline StackSmem stack_smem(int d, uint32_t slot_bytes, uint32_t r1_bytes) {
  StackSmem S{};
  S.ring = 0;
  S.r1 = static_cast<size_t>(kSlots) * slot_bytes;
  S.gam = S.r1 + r1_bytes;
  S.xs = S.gam + static_cast<size_t>(d) * 4;
  S.ctrl = S.xs + static_cast<size_t>(d) * 4;
  S.total = S.ctrl + sizeof(StackCtrl);
  return S;
}

// Rows per block: as many as fit kSlotTarget bytes, 1..7.
__host__ __device__ inline int rows_per_block(int row_bytes) {
  const int r = static_cast<int>(kSlotTarget) / row_bytes;
  return r < 1 ? 1 : (r > kConsumers ? kConsumers : r);
}

// A ring slot holds a phase-A block (ra rows of 2 d bytes) or a phase-B block (rb rows of 2 f bytes).
inline uint32_t slot_bytes_for(int d, int f) {
  const uint32_t a = static_cast<uint32_t>(rows_per_block(2 * d)) * 2u * d;
  const uint32_t b = static_cast<uint32_t>(rows_per_block(2 * f)) * 2u * f;
  return ((a > b ? a : b) + 127u) & ~127u;
}

// R1 holds a layer's router rows (E d bf16) during routing and h of the chosen experts (kMaxK f f32) in
// phase B.
inline uint32_t r1_bytes_for(int E_max, int d, int f) {
  const uint32_t wr = static_cast<uint32_t>(E_max) * d * 2u, hb = static_cast<uint32_t>(kMaxK) * f * 4u;
  return ((wr > hb ? wr : hb) + 15u) & ~15u;
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait(bar, parity, abort, kTimeoutNs);
}

__device__ __forceinline__ void abort_cta(StackCtrl& C, unsigned int* timeouts) {
  if (atomicExch(&C.abort, 1) == 0 && timeouts) atomicAdd(timeouts, 1u);
}

// Dot product of a bf16 row in shared memory with an f32 vector in shared memory over n elements
// (n % 8 == 0), by one warp; every lane returns the result.  Lane l takes the 8-element chunks
// [l 8 + 256 j, + 8) into four partial sums (chunk j into sum j mod 4: four short dependency chains
// instead of one long one), adds them as (s0 + s1) + (s2 + s3), then the warp in a fixed butterfly.
__device__ __forceinline__ float warp_dot(const uint16_t* row, const float* v, int n, int lane) {
  float p[4] = {0.f, 0.f, 0.f, 0.f};
  int j = 0;
  for (int c = lane * 8; c < n; c += 256, ++j) {
    float w[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(row + c), w);
    const float4 a = *reinterpret_cast<const float4*>(v + c);
    const float4 b = *reinterpret_cast<const float4*>(v + c + 4);
    const int q = j & 3;
    float acc = q == 0 ? p[0] : (q == 1 ? p[1] : (q == 2 ? p[2] : p[3]));
    acc = fmaf(w[0], a.x, acc);
    acc = fmaf(w[1], a.y, acc);
    acc = fmaf(w[2], a.z, acc);
    acc = fmaf(w[3], a.w, acc);
    acc = fmaf(w[4], b.x, acc);
    acc = fmaf(w[5], b.y, acc);
    acc = fmaf(w[6], b.z, acc);
    acc = fmaf(w[7], b.w, acc);
    if (q == 0) p[0] = acc;
    else if (q == 1) p[1] = acc;
    else if (q == 2) p[2] = acc;
    else p[3] = acc;
  }
  float acc = (p[0] + p[1]) + (p[2] + p[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// The same dot product with the vector held in registers: xr[j] = v[lane 8 + 256 j .. + 8) for the
// j < kXChunks chunks that lie below n (n <= 256 kXChunks).  Same summation order as warp_dot.
constexpr int kXChunks = 8;   // d <= 2048 keeps x in registers
__device__ __forceinline__ float warp_dot_xr(const uint16_t* row, const float (&xr)[kXChunks][8], int n, int lane) {
  float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < kXChunks; ++j) {
    const int c = lane * 8 + j * 256;
    if (c < n) {
      float w[8];
      unpack_bf16x8(*reinterpret_cast<const uint4*>(row + c), w);
#pragma unroll
      for (int i = 0; i < 8; ++i) p[j & 3] = fmaf(w[i], xr[j][i], p[j & 3]);
    }
  }
  float acc = (p[0] + p[1]) + (p[2] + p[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// v[c .. c + 8) from shared memory as two 16-byte loads (zeros when c >= n).
__device__ __forceinline__ void load_chunk8(const float* v, int c, int n, float (&out)[8]) {
  if (c < n) {
    const float4 a = *reinterpret_cast<const float4*>(v + c);
    const float4 b = *reinterpret_cast<const float4*>(v + c + 4);
    out[0] = a.x; out[1] = a.y; out[2] = a.z; out[3] = a.w;
    out[4] = b.x; out[5] = b.y; out[6] = b.z; out[7] = b.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = 0.f;
  }
}

// The same for phase B's h (f <= 256 kHChunks).
constexpr int kHChunks = 12;   // f <= 3072 keeps h in registers
__device__ __forceinline__ float warp_dot_hr(const uint16_t* row, const float (&hr)[kHChunks][8], int n, int lane) {
  float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int j = 0; j < kHChunks; ++j) {
    const int c = lane * 8 + j * 256;
    if (c < n) {
      float w[8];
      unpack_bf16x8(*reinterpret_cast<const uint4*>(row + c), w);
#pragma unroll
      for (int i = 0; i < 8; ++i) p[j & 3] = fmaf(w[i], hr[j][i], p[j & 3]);
    }
  }
  float acc = (p[0] + p[1]) + (p[2] + p[3]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// Warp reduce-scatter of 16 per-lane values p[0..16): on return lane l holds in p[0] the warp's sum of
// value l >> 1 (both lanes of a pair hold it).  Five steps of lane distance 16, 8, 4, 2, 1; at each the
// lane keeps the half of its values that its lane bit selects and adds the partner's copy of that half,
// so every sum is formed once, in a fixed order.
__device__ __forceinline__ float warp_reduce_scatter16(float (&p)[16], int lane) {
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const bool hi = (lane & 16) != 0;
    const float send = hi ? p[i] : p[i + 8], keep = hi ? p[i + 8] : p[i];
    p[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const bool hi = (lane & 8) != 0;
    const float send = hi ? p[i] : p[i + 4], keep = hi ? p[i + 4] : p[i];
    p[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const bool hi = (lane & 4) != 0;
    const float send = hi ? p[i] : p[i + 2], keep = hi ? p[i + 2] : p[i];
    p[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  }
  {
    const bool hi = (lane & 2) != 0;
    const float send = hi ? p[0] : p[1], keep = hi ? p[1] : p[0];
    p[0] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
  }
  return p[0] + __shfl_xor_sync(0xffffffffu, p[0], 1);
}

// Order-preserving map of a float onto uint32 (larger float -> larger key; -0 maps like +0).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t u = __float_as_uint(f + 0.f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The inverse of order_key.
__device__ __forceinline__ float key_float(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// Sum over the CTA (all threads take part); every thread receives the total.
__device__ __forceinline__ float cta_sum(float v, float* red) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float t = 0.f;
  for (int w = 0; w < kThreads / 32; ++w) t += red[w];
  __syncthreads();   // red is reused by the next sum
  return t;
}

// One producer thread: stages layer l's router rows and gain on C.st.
__device__ __forceinline__ void stage_layer(const StackArgs& a, int l, StackCtrl& C, unsigned char* wr_s,
                                            unsigned char* gam_s) {
  const StackLayerDev& Ly = a.L[l];
  const uint32_t wb = Ly.w_r ? static_cast<uint32_t>(Ly.E) * a.d * 2u : 0u;
  const uint32_t gb = static_cast<uint32_t>(a.d) * 4u;
  mbar_expect_tx(&C.st, wb + gb);
  for (uint32_t o = 0; o < wb; o += 32768u)
    bulk_load(wr_s + o, reinterpret_cast<const unsigned char*>(Ly.w_r) + o, wb - o < 32768u ? wb - o : 32768u, &C.st);
  for (uint32_t o = 0; o < gb; o += 32768u)
    bulk_load(gam_s + o, reinterpret_cast<const unsigned char*>(Ly.gamma) + o, gb - o < 32768u ? gb - o : 32768u,
              &C.st);
}

// Grid barrier among the consumer threads of all CTAs, run by one thread: arrival, then wait for
// `target` arrivals in total.  False on timeout or abort.
__device__ __forceinline__ bool grid_wait(unsigned int* gbar, unsigned int target, volatile int* abort) {
  red_release_add(gbar, 1u);
  const uint64_t t0 = globaltimer();
  for (uint32_t it = 0;; ++it) {
    if (ld_acquire(gbar) >= target) return true;
    if ((it & 15) == 15 && (*abort || globaltimer() - t0 > kTimeoutNs)) return false;
  }
}

__global__ void __launch_bounds__(kThreads, 1) stack_kernel(const __grid_constant__ StackArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int d = a.d, f = a.f;
  const StackSmem S = stack_smem(d, a.slot_bytes, a.r1_bytes);
  StackCtrl& C = *reinterpret_cast<StackCtrl*>(base + S.ctrl);
  unsigned char* wr_s = base + S.r1;                    // router rows (routing) ...
  float* hs = reinterpret_cast<float*>(base + S.r1);    // ... then h of the chosen experts (phase B)
  unsigned char* gam_s = base + S.gam;
  const float* gam = reinterpret_cast<const float*>(gam_s);
  float* xs = reinterpret_cast<float*>(base + S.xs);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nC = gridDim.x, c = blockIdx.x;
  volatile int* abort_flag = &C.abort;

  // this CTA's rows, the same in every layer
  const int f0 = static_cast<int>(static_cast<long long>(f) * c / nC);
  const int f1 = static_cast<int>(static_cast<long long>(f) * (c + 1) / nC);
  const int n0 = static_cast<int>(static_cast<long long>(d) * c / nC);
  const int n1 = static_cast<int>(static_cast<long long>(d) * (c + 1) / nC);
  const int nRA = f1 - f0, nRB = n1 - n0;
  const int RA = a.ra, RB = a.rb;
  const int GA = (nRA + RA - 1) / RA, GB = (nRB + RB - 1) / RB;   // blocks per chosen expert
  const int nvec = d / 8;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], kConsumers);   // one arrival per consumer warp
    }
    mbar_init(&C.st, 1);
    mbar_init(&C.hb, 1);
    mbar_init(&C.r1free, 1);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    stage_layer(a, 0, C, wr_s, gam_s);
  }
  if (a.ids && threadIdx.x < a.N) {
    int id = a.ids[threadIdx.x];
    if (id < 0 || id >= a.V) {
      if (c == 0) record_device_error(a.errors);
      id = -1;
    }
    C.ids[threadIdx.x] = id;
  }
  __syncthreads();

  // the residual stream entering layer 0, this thread's 8-element vectors v = threadIdx.x + j kThreads
  float hv[kMaxVec][8];
  if (a.ids) {
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxVec; ++j) {
      const int v = threadIdx.x + j * kThreads;
#pragma unroll
      for (int i = 0; i < 8; ++i) hv[j][i] = 0.f;
      if (v < nvec) {
        for (int cb = 0; cb < a.N; ++cb) {
          const int id = C.ids[cb];
          if (id < 0) continue;
          float w[8];
          unpack_bf16x8(*reinterpret_cast<const uint4*>(a.tables + (static_cast<size_t>(cb) * a.V + id) * d + v * 8), w);
#pragma unroll
          for (int i = 0; i < 8; ++i) hv[j][i] += w[i];
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += hv[j][i] * hv[j][i];
      }
    }
    const float inv = rsqrtf(cta_sum(ss, C.red) / static_cast<float>(d) + a.eps);
#pragma unroll
    for (int j = 0; j < kMaxVec; ++j) {
      const int v = threadIdx.x + j * kThreads;
      if (v >= nvec) continue;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int n = v * 8 + i;
        hv[j][i] = hv[j][i] * inv * __ldg(a.gamma0 + n);
        if (n >= n0 && n < n1) a.h[n] = hv[j][i];   // this CTA's rows of the stream, updated in phase B
      }
    }
  }

  bool ok = true;
  int q = 0;               // ring items of the layers so far (every thread keeps the same count)
  int issued = 0;          // producer: items armed on `full`
  int staged = 1;          // producer: layers staged on C.st
  int h_armed = 0;         // thread 32: layers whose h copy was armed on C.hb
  const int L = a.n_layers;
  for (int l = 0; l < L; ++l) {
    const StackLayerDev& Ly = a.L[l];
    const int E = Ly.E, k = Ly.k;
    // ---- this layer's router rows and gain are staged ----
    ok = __syncthreads_and(ok && wait_bounded(&C.st, static_cast<uint32_t>(l & 1), abort_flag));
    if (!ok) {
      if (threadIdx.x == 0) abort_cta(C, a.timeouts);
      break;
    }
    // the layer's biases, loaded alongside the residual stream (read after the norm's CTA barriers)
    if (threadIdx.x < E) {
      C.qb[threadIdx.x] = Ly.logit_bias ? Ly.logit_bias[threadIdx.x] : 0.f;
      C.sb[threadIdx.x] = Ly.sel_bias ? Ly.sel_bias[threadIdx.x] : 0.f;
    }
    // ---- pre-norm: x = bf16(RMSNorm(h) * gamma), kept as f32 in hv (this thread's vectors) and xs ----
    if (l > 0 || !a.ids) {
#pragma unroll
      for (int j = 0; j < kMaxVec; ++j) {
        const int v = threadIdx.x + j * kThreads;
        if (v < nvec) {
          const float4 p0 = __ldcg(reinterpret_cast<const float4*>(a.h + v * 8));
          const float4 p1 = __ldcg(reinterpret_cast<const float4*>(a.h + v * 8 + 4));
          hv[j][0] = p0.x; hv[j][1] = p0.y; hv[j][2] = p0.z; hv[j][3] = p0.w;
          hv[j][4] = p1.x; hv[j][5] = p1.y; hv[j][6] = p1.z; hv[j][7] = p1.w;
        }
      }
    }
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < kMaxVec; ++j)
      if (threadIdx.x + j * kThreads < nvec)
#pragma unroll
        for (int i = 0; i < 8; ++i) ss += hv[j][i] * hv[j][i];
    const float inv = rsqrtf(cta_sum(ss, C.red) / static_cast<float>(d) + a.eps);
#pragma unroll
    for (int j = 0; j < kMaxVec; ++j) {
      const int v = threadIdx.x + j * kThreads;
      if (v >= nvec) continue;
      float g[8];
      load_chunk8(gam, v * 8, d, g);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int n = v * 8 + i;
        const uint16_t b = f32_to_bf16_bits(hv[j][i] * inv * g[i]);
        if (c == 0 && a.layer_x) a.layer_x[static_cast<size_t>(l) * d + n] = b;
        if (c == 0 && a.layer_h) a.layer_h[static_cast<size_t>(l) * d + n] = hv[j][i];
        hv[j][i] = bf16_to_f32(b);
      }
      *reinterpret_cast<float4*>(xs + v * 8) = make_float4(hv[j][0], hv[j][1], hv[j][2], hv[j][3]);
      *reinterpret_cast<float4*>(xs + v * 8 + 4) = make_float4(hv[j][4], hv[j][5], hv[j][6], hv[j][7]);
    }
    // ---- router logits: each thread's dot products over its own vectors of x, 16 experts at a time, a
    // reduce-scatter per warp, then (warp 0, below) the 8 warps' partial sums in warp order ----
    if (Ly.w_r) {
      const uint16_t* wr = reinterpret_cast<const uint16_t*>(wr_s);
      for (int e0 = 0; e0 < E; e0 += 16) {
        float pl[16];
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          pl[t] = 0.f;
          if (e0 + t < E) {
#pragma unroll
            for (int j = 0; j < kMaxVec; ++j) {
              const int v = threadIdx.x + j * kThreads;
              if (v < nvec) {
                float w[8];
                unpack_bf16x8(*reinterpret_cast<const uint4*>(wr + static_cast<size_t>(e0 + t) * d + v * 8), w);
#pragma unroll
                for (int i = 0; i < 8; ++i) pl[t] = fmaf(w[i], hv[j][i], pl[t]);
              }
            }
          }
        }
        const float s = warp_reduce_scatter16(pl, lane);
        if ((lane & 1) == 0 && e0 + (lane >> 1) < E) C.lpart[warp][e0 + (lane >> 1)] = s;
      }
    }
    __syncthreads();
    // ---- top-k (larger score first, ties to the lower index) and gates, by warp 0: lane l holds experts
    // l and l + 32; maxima and arg-maxima by warp reductions, the softmax sum by a butterfly ----
    if (warp == 0) {
      if (!Ly.w_r) {
        if (lane == 0) {
          C.uexp[0] = 0;
          C.gsel[0] = 1.f;
          C.nu = 1;
        }
      } else {
        // scores as order-preserving keys (0: no expert; 1: a NaN score, chosen only when nothing else is
        // left), so that each choice is a warp max then a warp min of the expert index among the maxima
        float qv[2];
        uint32_t sk[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int e = lane + 32 * j;
          float lg = 0.f;
          if (e < E) {
#pragma unroll
            for (int w = 0; w < kThreads / 32; ++w) lg += C.lpart[w][e];
          }
          qv[j] = e < E ? lg + C.qb[e] : -INFINITY;
          const float sv = e < E ? qv[j] + C.sb[e] : 0.f;
          sk[j] = e >= E ? 0u : (sv != sv ? 1u : order_key(sv));
        }
        const uint32_t qk = max(qv[0] != qv[0] ? 0u : order_key(qv[0]), qv[1] != qv[1] ? 0u : order_key(qv[1]));
        const float m = key_float(__reduce_max_sync(0xffffffffu, qk));   // the largest logit (NaN ignored)
        float z = (lane < E ? expf(qv[0] - m) : 0.f) + (lane + 32 < E ? expf(qv[1] - m) : 0.f);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
        int sel[kMaxK];
        float qsel[kMaxK];
#pragma unroll
        for (int i = 0; i < kMaxK; ++i) {
          if (i >= k) break;
          const bool hi = sk[1] > sk[0];   // the lane's best (its lower expert on a tie)
          const uint32_t kb = hi ? sk[1] : sk[0];
          const uint32_t mk = __reduce_max_sync(0xffffffffu, kb);
          const int be = static_cast<int>(
              __reduce_min_sync(0xffffffffu, kb == mk ? static_cast<uint32_t>(hi ? lane + 32 : lane) : 0xffffu));
          sel[i] = be;
          qsel[i] = __shfl_sync(0xffffffffu, (be >> 5) ? qv[1] : qv[0], be & 31);
          if ((be & 31) == lane) {   // not chosen twice
            if (be >> 5) sk[1] = 0u;
            else sk[0] = 0u;
          }
        }
        if (lane == 0) {
          if (k == 1) {
            C.uexp[0] = sel[0];
            C.gsel[0] = expf(qsel[0] - m) / z;
            C.nu = 1;
          } else {
            const float z1 = expf(qsel[0] - m), z2 = expf(qsel[1] - m);
            const float iz = 1.f / (z1 + z2);
            C.uexp[0] = sel[0];
            C.gsel[0] = z1 * iz;
            C.uexp[1] = sel[1];
            C.gsel[1] = z2 * iz;
            C.nu = 2;
          }
        }
      }
      __syncwarp();
      if (c == 0 && lane == 0) {
        for (int i = 0; i < kMaxK; ++i) {
          if (a.layer_idx) a.layer_idx[l * kMaxK + i] = i < C.nu ? C.uexp[i] : -1;
          if (a.layer_gates) a.layer_gates[l * kMaxK + i] = i < C.nu ? C.gsel[i] : 0.f;
        }
      }
    }
    // the staging area and xs were accessed through the generic proxy; bulk copies follow
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    const int nu = C.nu;
    // items of this layer: phase A, per chosen expert u and block g, a gate block then an up block
    // (i = 2 (u GA + g) + {0, 1}); phase B, per u and g, a W_down block (i = nA + u GB + g)
    const int nA = 2 * nu * GA, nIt = nA + nu * GB;

    if (warp == 0) {
      // ================================ producer ================================
      if (lane == 0) {
        int i = 0;
        for (; i < nIt; ++i) {
          const int qq = q + i, slot = qq % kSlots;
          if (!wait_bounded(&C.empty[slot], static_cast<uint32_t>((qq / kSlots) & 1) ^ 1u, abort_flag)) break;
          unsigned char* dst = base + static_cast<size_t>(slot) * a.slot_bytes;
          const uint16_t* src;
          uint32_t bytes;
          if (i < nA) {
            const int blk = i >> 1, u = blk / GA, r0 = f0 + (blk % GA) * RA;
            const int nr = (f1 - r0) < RA ? (f1 - r0) : RA;
            src = ((i & 1) ? Ly.w_up : Ly.w_gate) + (static_cast<size_t>(C.uexp[u]) * f + r0) * d;
            bytes = static_cast<uint32_t>(nr) * d * 2u;
          } else {
            const int j = i - nA, u = j / GB, m0 = n0 + (j % GB) * RB;
            const int nr = (n1 - m0) < RB ? (n1 - m0) : RB;
            src = Ly.w_down + (static_cast<size_t>(C.uexp[u]) * d + m0) * f;
            bytes = static_cast<uint32_t>(nr) * f * 2u;
          }
          mbar_expect_tx(&C.full[slot], bytes);
          bulk_load(dst, src, bytes, &C.full[slot]);
        }
        issued = q + i;
        if (i < nIt) {
          abort_cta(C, a.timeouts);
        } else if (l + 1 < L) {
          // the next layer's router rows go where phase B reads h: wait until it has
          if (wait_bounded(&C.r1free, static_cast<uint32_t>(l & 1), abort_flag)) {
            stage_layer(a, l + 1, C, wr_s, gam_s);
            ++staged;
          } else {
            abort_cta(C, a.timeouts);
          }
        }
      }
      __syncwarp();
    } else {
      // ================================ consumers (warps 1..7) ================================
      // every consumer warp takes every item in order; warp cw contracts row cw of the block
      const int cw = warp - 1;
      // x in registers for the phase-A dot products (when d fits kXChunks chunks), loaded while the
      // first block is in flight
      const bool x_in_regs = d <= 256 * kXChunks;
      float xr[kXChunks][8];
#pragma unroll
      for (int j = 0; j < kXChunks; ++j) load_chunk8(xs, lane * 8 + j * 256, x_in_regs ? d : 0, xr[j]);
      // phase A: h of the owned f-rows of each chosen expert
      for (int i = 0; i < nA && ok; ++i) {
        const int qq = q + i, slot = qq % kSlots;
        ok = __all_sync(0xffffffffu, wait_bounded(&C.full[slot], static_cast<uint32_t>((qq / kSlots) & 1), abort_flag));
        if (!ok) break;
        const int blk = i >> 1, u = blk / GA, r0 = f0 + (blk % GA) * RA;
        const int nr = (f1 - r0) < RA ? (f1 - r0) : RA;
        if (cw < nr) {
          const uint16_t* row = reinterpret_cast<const uint16_t*>(base + static_cast<size_t>(slot) * a.slot_bytes) +
                                static_cast<size_t>(cw) * d;
          const float v = x_in_regs ? warp_dot_xr(row, xr, d, lane) : warp_dot(row, xs, d, lane);
          if ((i & 1) == 0) {
            if (lane == 0) C.gv[cw] = v;                     // the gate value waits for the up block
          } else if (lane == 0) {
            const float gv = C.gv[cw];
            a.hbuf[static_cast<size_t>(u) * f + r0 + cw] = gv / (1.f + expf(-gv)) * v;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[slot]);
      }
      // grid barrier 1: every CTA's h rows are stored
      ok = bar_and(1, kConsumers * 32, ok);
      if (threadIdx.x == 32) {
        const bool passed = ok && grid_wait(a.gbar, static_cast<unsigned int>(2 * l + 1) * nC, abort_flag);
        if (passed) {
          // h was written through the generic proxy by other CTAs: order it before the bulk copy
          asm volatile("fence.proxy.async.global;" ::: "memory");
          const uint32_t hbytes = static_cast<uint32_t>(nu) * f * 4u;
          mbar_expect_tx(&C.hb, hbytes);
          ++h_armed;
          for (uint32_t o = 0; o < hbytes; o += 32768u)
            bulk_load(reinterpret_cast<unsigned char*>(hs) + o, reinterpret_cast<const unsigned char*>(a.hbuf) + o,
                      hbytes - o < 32768u ? hbytes - o : 32768u, &C.hb);
        } else {
          abort_cta(C, a.timeouts);
        }
      }
      ok = bar_and(1, kConsumers * 32, ok && !*abort_flag);
      if (ok) ok = __all_sync(0xffffffffu, wait_bounded(&C.hb, static_cast<uint32_t>(l & 1), abort_flag));
      // phase B: the owned d-rows of each chosen expert; this expert's h in registers when f fits
      const bool h_in_regs = f <= 256 * kHChunks;
      float hr[kHChunks][8];
      int hr_u = -1;
      for (int i = nA; i < nIt && ok; ++i) {
        const int qq = q + i, slot = qq % kSlots;
        ok = __all_sync(0xffffffffu, wait_bounded(&C.full[slot], static_cast<uint32_t>((qq / kSlots) & 1), abort_flag));
        if (!ok) break;
        const int j = i - nA, u = j / GB, m = (j % GB) * RB;        // m: first row, relative to n0
        const int nr = (nRB - m) < RB ? (nRB - m) : RB;
        if (h_in_regs && u != hr_u) {
          const float* hu = hs + static_cast<size_t>(u) * f;
#pragma unroll
          for (int jj = 0; jj < kHChunks; ++jj) load_chunk8(hu, lane * 8 + jj * 256, f, hr[jj]);
          hr_u = u;
        }
        if (cw < nr) {
          const uint16_t* row = reinterpret_cast<const uint16_t*>(base + static_cast<size_t>(slot) * a.slot_bytes) +
                                static_cast<size_t>(cw) * f;
          const float v = h_in_regs ? warp_dot_hr(row, hr, f, lane)
                                    : warp_dot(row, hs + static_cast<size_t>(u) * f, f, lane);
          if (lane == 0) C.ypart[u][m + cw] = v;
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.empty[slot]);
      }
      // h (in the router rows' area) has been read: the producer may stage the next layer there
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      ok = bar_and(1, kConsumers * 32, ok);
      if (threadIdx.x == 32 && ok) mbar_arrive(&C.r1free);
      // the owned rows of the residual stream: h + the chosen experts in slot order
      if (ok) {
        for (int n = threadIdx.x - 32; n < nRB; n += kConsumers * 32) {
          float acc = 0.f;
          for (int u = 0; u < nu; ++u) acc = fmaf(C.gsel[u], C.ypart[u][n], acc);
          a.h[n0 + n] = __ldcg(a.h + n0 + n) + acc;
        }
      }
      // grid barrier 2: the whole stream is updated (not after the last layer: the launch's end is)
      ok = bar_and(1, kConsumers * 32, ok);
      if (l + 1 < L && threadIdx.x == 32) {
        if (!(ok && grid_wait(a.gbar, static_cast<unsigned int>(2 * l + 2) * nC, abort_flag))) abort_cta(C, a.timeouts);
      }
    }
    q += nIt;
    ok = __syncthreads_and(ok && !*abort_flag);
    if (!ok) {
      if (threadIdx.x == 0) abort_cta(C, a.timeouts);
      break;
    }
  }
  __syncthreads();

  // after an abort: copies still landing in shared memory must land before the CTA goes (bounded)
  if (*abort_flag) {
    if (threadIdx.x == 0) {
      for (int s = 0; s < kSlots && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / kSlots) * kSlots;
        const uint64_t t1 = globaltimer();
        while (!mbar_try_wait(&C.full[s], static_cast<uint32_t>((last / kSlots) & 1)) &&
               globaltimer() - t1 < kTimeoutNs) {
        }
      }
      const uint64_t t1 = globaltimer();
      while (!mbar_try_wait(&C.st, static_cast<uint32_t>((staged - 1) & 1)) && globaltimer() - t1 < kTimeoutNs) {
      }
    }
    if (threadIdx.x == 32 && h_armed > 0) {
      const uint64_t t1 = globaltimer();
      while (!mbar_try_wait(&C.hb, static_cast<uint32_t>((h_armed - 1) & 1)) && globaltimer() - t1 < kTimeoutNs) {
      }
    }
  }
  __syncwarp();
  __syncthreads();
}

}  // namespace
}  // namespace zmoe

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------
extern "C" {

size_t zmoe_decode_stack_workspace_size(int n_layers, int d, int f, int E_max) {
  using namespace zmoe;
  if (n_layers < 1 || n_layers > kMaxLayers || d < 8 || d % 8 != 0 || d > 8 * kThreads * kMaxVec || f < 8 ||
      f % 8 != 0 || E_max < 1 || E_max > kMaxE)
    return 0;
  const int nC = num_sms();
  if (nC < 1 || (d + nC - 1) / nC > kMaxRowsB ||
      stack_smem(d, slot_bytes_for(d, f), r1_bytes_for(E_max, d, f)).total + 1024 >
          static_cast<size_t>(max_smem_optin()))
    return 0;
  return 256 + static_cast<size_t>(kMaxK) * f * 4;
}

zmoe_status zmoe_decode_stack(const zmoe_stack_layer* layers, int n_layers, int d, int f, float eps,
                              const int32_t* ids, const void* tables, const float* gamma0, int N, int V, float* h,
                              int32_t* layer_idx, float* layer_gates, float* layer_h, void* layer_x, void* workspace,
                              size_t ws_bytes, zmoe_stream_t stream) {
  ZMOE_TRACE("zmoe_decode_stack");
  using namespace zmoe;
  ZMOE_REQUIRE(layers && n_layers >= 1 && n_layers <= kMaxLayers, "zmoe_decode_stack: n_layers must be in [1, 32]");
  ZMOE_REQUIRE(d >= 8 && d % 8 == 0 && d <= 8 * kThreads * kMaxVec && f >= 8 && f % 8 == 0,
               "zmoe_decode_stack: d must be a multiple of 8 in [8, 4096], f a multiple of 8");
  ZMOE_REQUIRE(eps >= 0.f, "zmoe_decode_stack: eps must be >= 0");
  ZMOE_REQUIRE(h && aligned16(h), "zmoe_decode_stack: h must be a 16-byte aligned device pointer");
  if (ids) {
    ZMOE_REQUIRE(tables && gamma0 && N >= 1 && N <= kMaxN && V >= 1 && aligned16(tables),
                 "zmoe_decode_stack: with ids, tables (16-byte aligned), gamma0, N in [1, 32] and V >= 1 are needed");
  }
  ZMOE_REQUIRE(!layer_x || aligned16(layer_x), "zmoe_decode_stack: layer_x must be 16-byte aligned");
  StackArgs a{};
  int E_max = 1;
  for (int l = 0; l < n_layers; ++l) {
    const zmoe_stack_layer& Ly = layers[l];
    ZMOE_REQUIRE(Ly.E >= 1 && Ly.E <= kMaxE, "zmoe_decode_stack: a layer's E must be in [1, 64]");
    ZMOE_REQUIRE((Ly.k == 1 || Ly.k == 2) && Ly.k <= Ly.E, "zmoe_decode_stack: a layer's k must be 1 or 2 and <= E");
    ZMOE_REQUIRE(Ly.w_router || (Ly.E == 1 && Ly.k == 1),
                 "zmoe_decode_stack: w_router may be NULL only for a dense layer (E == 1)");
    ZMOE_REQUIRE(Ly.gamma && Ly.w_gate && Ly.w_up && Ly.w_down, "zmoe_decode_stack: NULL layer pointer");
    ZMOE_REQUIRE(aligned16(Ly.gamma) && aligned16(Ly.w_gate) && aligned16(Ly.w_up) && aligned16(Ly.w_down) &&
                     (!Ly.w_router || aligned16(Ly.w_router)),
                 "zmoe_decode_stack: layer pointers must be 16-byte aligned");
    StackLayerDev& D = a.L[l];
    D.w_r = static_cast<const uint16_t*>(Ly.w_router);
    D.logit_bias = Ly.logit_bias;
    D.sel_bias = Ly.sel_bias;
    D.gamma = Ly.gamma;
    D.w_gate = static_cast<const uint16_t*>(Ly.w_gate);
    D.w_up = static_cast<const uint16_t*>(Ly.w_up);
    D.w_down = static_cast<const uint16_t*>(Ly.w_down);
    D.E = Ly.E;
    D.k = Ly.k;
    if (Ly.w_router && Ly.E > E_max) E_max = Ly.E;
  }
  const uint32_t r1 = r1_bytes_for(E_max, d, f);
  const int nC = num_sms();
  const uint32_t slot = slot_bytes_for(d, f);
  const StackSmem S = stack_smem(d, slot, r1);
  const size_t smem = S.total + 1024;
  if (nC < 1 || (d + nC - 1) / nC > kMaxRowsB || smem > static_cast<size_t>(max_smem_optin()))
    return fail(ZMOE_ERR_UNSUPPORTED, "zmoe_decode_stack: these sizes do not fit one SM's shared memory");
  const size_t need = 256 + static_cast<size_t>(kMaxK) * f * 4;
  if (!workspace || ws_bytes < need)
    return fail(ZMOE_ERR_WORKSPACE_TOO_SMALL,
                "zmoe_decode_stack: workspace smaller than zmoe_decode_stack_workspace_size()");
  clear_error();
  a.n_layers = n_layers;
  a.d = d;
  a.f = f;
  a.N = N;
  a.V = V;
  a.eps = eps;
  a.ids = ids;
  a.tables = static_cast<const uint16_t*>(tables);
  a.gamma0 = gamma0;
  a.h = h;
  unsigned char* w = static_cast<unsigned char*>(workspace);
  a.gbar = reinterpret_cast<unsigned int*>(w);
  a.hbuf = reinterpret_cast<float*>(w + 256);
  a.timeouts = device_timeout_counter();
  a.errors = device_error_counter();
  a.layer_idx = layer_idx;
  a.layer_gates = layer_gates;
  a.layer_h = layer_h;
  a.layer_x = static_cast<uint16_t*>(layer_x);
  a.slot_bytes = slot;
  a.r1_bytes = r1;
  a.ra = rows_per_block(2 * d);
  a.rb = rows_per_block(2 * f);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, 256, s) != cudaSuccess)
    return check_launch("zmoe_decode_stack: clearing the barrier");
  if (cudaFuncSetAttribute(stack_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return check_launch("zmoe_decode_stack");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(nC));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: they wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, stack_kernel, a);
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string("zmoe_decode_stack: ") + cudaGetErrorString(e));
  return check_launch("zmoe_decode_stack");
}

}  // extern "C"
