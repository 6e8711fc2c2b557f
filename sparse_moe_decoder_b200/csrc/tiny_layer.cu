// The MoE layer at batch sizes of a few tokens (T * k <= 4): one cooperative launch without split-k.
//
// Same layer as zmoe_moe_layer (ZONOS2 digest items 5-6; the telknet.cc article on ZONOS2, section
// 2.1): the optional pre-norm x = bf16(RMSNorm(h) * gamma), router logits, top-k and gates, and
//   y[t] = h[t] + sum_i gate[t, i] * W_down[e] (silu(W_gate[e] x[t]) * (W_up[e] x[t])),  e = e(t, i).
//
// With one or two tokens the layer is a few matrix-vector products, and the weights of the chosen
// experts (37.75 MB each at d = 2048, f = 3072) are the only bytes that matter.  The stream-K tensor
// core kernel splits every weight row over several SMs at this size, and its partial sums and
// hand-offs between SMs cost more than the streaming.  Here every weight row is contracted whole on
// one SM, on the CUDA cores:
//   * every CTA repeats the pre-norm, the router logits (all E rows, staged by bulk copy) and the
//     selection, so no grid barrier precedes the weights;
//   * phase A: CTA c owns the f-rows [c f / C, (c + 1) f / C) of every chosen expert; one gate row and
//     one up row per ring slot (bulk copies into a ring of shared-memory slots, one producer thread),
//     a warp per slot, and h of the owned rows goes to global memory in fp32;
//   * one grid barrier (only the consumers take part: the producer keeps streaming W_down rows);
//   * phase B: CTA c owns the d-rows [c d / C, (c + 1) d / C); it bulk-loads all of h and contracts
//     its W_down rows, then writes y for its rows, summing the chosen experts in slot order.
// Every sum is fp32 and in a fixed order (no atomics): the result does not depend on timing.
#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int kThreads = 256;          // warp 0: producer; warps 1..7: consumers
constexpr int kConsumers = 7;
constexpr int kMaxA = 4;               // assignments T * k
// Slot s is always consumed by warp 1 + s % kConsumers, so each slot's phases are waited on in order by
// one warp (a waiter that ran a phase ahead of its slot would read a stale parity as done).
constexpr int kSlots = 2 * kConsumers;
static_assert(kSlots % kConsumers == 0, "a slot must belong to one consumer warp");
constexpr int kMaxE = 64;
constexpr int kMaxRowsB = 64;          // d-rows per CTA
constexpr unsigned long long kTimeoutNs = 2000000000ull;

struct TinyArgs {
  const uint16_t* x_in;    // [T, d] (without gamma)
  const float* h_in;       // [T, d] residual stream (input of the pre-norm with gamma; residual either way)
  const float* gamma;      // [d] or null
  float eps;
  const uint16_t* w_r;     // [E, d] or null (E == 1)
  const float* logit_bias;
  const float* sel_bias;
  const uint16_t* w_gate;  // [E, f, d]
  const uint16_t* w_up;    // [E, f, d]
  const uint16_t* w_down;  // [E, d, f]
  int T, d, f, E, k;
  float* y;                // [T, d]
  int32_t* expert_idx;     // [T, k] or null
  float* gates;            // [T, k] or null
  float* margin;           // [T] or null
  uint16_t* x_norm;        // [T, d] or null
  float* hbuf;             // [T k, f] workspace
  unsigned int* gbar;      // workspace, zeroed before the launch
  unsigned int* timeouts;
  uint32_t slot_bytes;     // max(4 d, 2 f), a multiple of 16
};

struct __align__(16) TinyCtrl {
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t st;             // staging: router rows, token rows, gamma
  uint64_t hb;             // h, after the grid barrier
  int abort;
  int ids[kMaxA];          // expert of assignment a = t k + i
  float gsel[kMaxA];       // its gate
  int nu;                  // distinct chosen experts, ascending
  int uexp[kMaxA];
  int ua[kMaxA][kMaxA];    // assignments of each chosen expert
  int una[kMaxA];
  float red[kThreads / 32];
  float logit[kMaxA * kMaxE];
  float ypart[kMaxA][kMaxRowsB];
};

// Shared memory: ring | xs [T][d] f32 | hs [T k][f] f32 | control.  The ring holds the staging copies
// (router rows, token rows, gamma) before the weights stream through it.
struct TinySmem {
  size_t ring, xs, hs, ctrl, total;
};

__host__ __device__ inline TinySmem tiny_smem(int T, int k, int d, int f, uint32_t slot_bytes) {
  TinySmem S{};
  S.ring = 0;
  S.xs = static_cast<size_t>(kSlots) * slot_bytes;
  S.hs = S.xs + static_cast<size_t>(T) * d * 4;
  S.ctrl = S.hs + static_cast<size_t>(T) * k * f * 4;
  S.total = S.ctrl + sizeof(TinyCtrl);
  return S;
}

__device__ __forceinline__ bool wait_bounded(uint64_t* bar, uint32_t parity, volatile int* abort) {
  return mbar_wait(bar, parity, abort, kTimeoutNs);
}

__device__ __forceinline__ void abort_cta(TinyCtrl& C, unsigned int* timeouts) {
  if (atomicExch(&C.abort, 1) == 0 && timeouts) atomicAdd(timeouts, 1u);
}

// Dot product of a bf16 row held in shared memory with an f32 vector in shared memory, over n
// elements (n % 8 == 0), by one warp: lane l takes the 8-element chunks l, l + 32, ...; the partial
// sums are combined by a butterfly, so every lane holds the result.
__device__ __forceinline__ float warp_dot(const uint16_t* row, const float* v, int n, int lane) {
  float acc = 0.f;
  for (int c = lane * 8; c < n; c += 256) {
    float w[8];
    unpack_bf16x8(*reinterpret_cast<const uint4*>(row + c), w);
    const float4 a = *reinterpret_cast<const float4*>(v + c);
    const float4 b = *reinterpret_cast<const float4*>(v + c + 4);
    acc = fmaf(w[0], a.x, acc);
    acc = fmaf(w[1], a.y, acc);
    acc = fmaf(w[2], a.z, acc);
    acc = fmaf(w[3], a.w, acc);
    acc = fmaf(w[4], b.x, acc);
    acc = fmaf(w[5], b.y, acc);
    acc = fmaf(w[6], b.z, acc);
    acc = fmaf(w[7], b.w, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

__global__ void __launch_bounds__(kThreads, 1) tiny_layer_kernel(TinyArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const TinySmem S = tiny_smem(a.T, a.k, a.d, a.f, a.slot_bytes);
  TinyCtrl& C = *reinterpret_cast<TinyCtrl*>(base + S.ctrl);
  float* xs = reinterpret_cast<float*>(base + S.xs);
  float* hs = reinterpret_cast<float*>(base + S.hs);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int T = a.T, d = a.d, f = a.f, E = a.E, k = a.k, nA = a.T * a.k;
  const int nC = gridDim.x, c = blockIdx.x;
  volatile int* abort_flag = &C.abort;

  // staging layout inside the ring: router rows, token rows, gamma
  uint16_t* wr_s = reinterpret_cast<uint16_t*>(base);
  const size_t wr_bytes = a.w_r ? static_cast<size_t>(E) * d * 2 : 0;
  unsigned char* tok_s = base + wr_bytes;
  const size_t tok_bytes = static_cast<size_t>(T) * d * (a.gamma ? 4 : 2);
  float* gam_s = reinterpret_cast<float*>(tok_s + tok_bytes);
  const size_t gam_bytes = a.gamma ? static_cast<size_t>(d) * 4 : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], 1);
    }
    mbar_init(&C.st, 1);
    mbar_init(&C.hb, 1);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_expect_tx(&C.st, static_cast<uint32_t>(wr_bytes + tok_bytes + gam_bytes));
    const unsigned char* src[3] = {reinterpret_cast<const unsigned char*>(a.w_r),
                                   a.gamma ? reinterpret_cast<const unsigned char*>(a.h_in)
                                           : reinterpret_cast<const unsigned char*>(a.x_in),
                                   reinterpret_cast<const unsigned char*>(a.gamma)};
    unsigned char* dst[3] = {base, tok_s, reinterpret_cast<unsigned char*>(gam_s)};
    const size_t len[3] = {wr_bytes, tok_bytes, gam_bytes};
    for (int i = 0; i < 3; ++i)
      for (size_t o = 0; o < len[i]; o += 32768) {
        const uint32_t n = static_cast<uint32_t>(len[i] - o < 32768 ? len[i] - o : 32768);
        bulk_load(dst[i] + o, src[i] + o, n, &C.st);
      }
  }
  __syncthreads();
  bool ok = __syncthreads_and(wait_bounded(&C.st, 0, abort_flag));

  // ---- the routed input rows x (f32 copies of bf16 values) ----
  if (ok) {
    for (int t = 0; t < T; ++t) {
      if (a.gamma) {
        const float* hr = reinterpret_cast<const float*>(tok_s) + static_cast<size_t>(t) * d;
        float ss = 0.f;
        for (int i = threadIdx.x * 4; i < d; i += kThreads * 4) {
          const float4 v = *reinterpret_cast<const float4*>(hr + i);
          ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (lane == 0) C.red[warp] = ss;
        __syncthreads();
        float tot = 0.f;
        for (int w = 0; w < kThreads / 32; ++w) tot += C.red[w];
        const float inv = rsqrtf(tot / static_cast<float>(d) + a.eps);
        for (int i = threadIdx.x; i < d; i += kThreads) {
          const uint16_t b = f32_to_bf16_bits(hr[i] * inv * gam_s[i]);
          xs[static_cast<size_t>(t) * d + i] = bf16_to_f32(b);
          if (c == 0 && a.x_norm) a.x_norm[static_cast<size_t>(t) * d + i] = b;
        }
        __syncthreads();   // C.red is reused by the next token
      } else {
        const uint16_t* xr = reinterpret_cast<const uint16_t*>(tok_s) + static_cast<size_t>(t) * d;
        for (int i = threadIdx.x; i < d; i += kThreads) xs[static_cast<size_t>(t) * d + i] = bf16_to_f32(xr[i]);
      }
    }
  }
  __syncthreads();

  // ---- router logits for every (token, expert), one warp per pair ----
  if (ok) {
    for (int pq = warp; pq < T * E; pq += kThreads / 32) {
      const int t = pq / E, e = pq % E;
      const float v = a.w_r ? warp_dot(wr_s + static_cast<size_t>(e) * d, xs + static_cast<size_t>(t) * d, d, lane) : 0.f;
      if (lane == 0) C.logit[pq] = v;
    }
  }
  __syncthreads();

  // ---- top-k and gates: larger score first, ties to the lower index; softmax over logit + bias ----
  if (ok && threadIdx.x < T) {
    const int t = threadIdx.x;
    const float NEG = -INFINITY;
    float s1 = NEG, s2 = NEG, s3 = NEG, q1 = NEG, q2 = NEG, m = NEG;
    int e1 = -1, e2 = -1;
    for (int e = 0; e < E; ++e) {
      const float q = C.logit[t * E + e] + (a.logit_bias ? a.logit_bias[e] : 0.f);
      const float sc = q + (a.sel_bias ? a.sel_bias[e] : 0.f);
      m = fmaxf(m, q);
      if (e1 < 0 || sc > s1) {
        s3 = s2;
        s2 = s1;
        e2 = e1;
        q2 = q1;
        s1 = sc;
        e1 = e;
        q1 = q;
      } else if (e2 < 0 || sc > s2) {
        s3 = s2;
        s2 = sc;
        e2 = e;
        q2 = q;
      } else if (sc > s3) {
        s3 = sc;
      }
    }
    float z = 0.f;
    for (int e = 0; e < E; ++e) z += expf(C.logit[t * E + e] + (a.logit_bias ? a.logit_bias[e] : 0.f) - m);
    float g1, g2 = 0.f, mg;
    if (k == 1) {
      g1 = expf(q1 - m) / z;
      mg = (E > 1) ? s1 - s2 : INFINITY;
    } else {
      const float z1 = expf(q1 - m), z2 = expf(q2 - m);
      const float inv = 1.f / (z1 + z2);
      g1 = z1 * inv;
      g2 = z2 * inv;
      mg = (E > 2) ? fminf(s1 - s2, s2 - s3) : s1 - s2;
    }
    C.ids[t * k] = e1;
    C.gsel[t * k] = g1;
    if (k == 2) {
      C.ids[t * k + 1] = e2;
      C.gsel[t * k + 1] = g2;
    }
    if (c == 0) {
      if (a.expert_idx) {
        a.expert_idx[t * k] = e1;
        if (k == 2) a.expert_idx[t * k + 1] = e2;
      }
      if (a.gates) {
        a.gates[t * k] = g1;
        if (k == 2) a.gates[t * k + 1] = g2;
      }
      if (a.margin) a.margin[t] = mg;
    }
  }
  __syncthreads();
  if (ok && threadIdx.x == 0) {
    // distinct experts in ascending order, each with its assignments
    int nu = 0;
    for (int e = 0; e < E; ++e) {
      int n = 0;
      for (int q = 0; q < nA; ++q)
        if (C.ids[q] == e) C.ua[nu][n++] = q;
      if (n > 0) {
        C.uexp[nu] = e;
        C.una[nu] = n;
        ++nu;
      }
    }
    C.nu = nu;
  }
  // the staging copies in the ring were read through the generic proxy; the weights' bulk copies follow
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();

  // the work of this CTA: phase A items (expert u, f-row r), then phase B items (expert u, d-row n)
  const int f0 = static_cast<int>(static_cast<long long>(f) * c / nC), f1 = static_cast<int>(static_cast<long long>(f) * (c + 1) / nC);
  const int n0 = static_cast<int>(static_cast<long long>(d) * c / nC), n1 = static_cast<int>(static_cast<long long>(d) * (c + 1) / nC);
  const int nu = ok ? C.nu : 0;
  const int nItA = nu * (f1 - f0), nIt = nItA + nu * (n1 - n0);

  if (warp == 0) {
    // ============================== producer ==============================
    if (lane == 0 && ok) {
      int i = 0;
      for (; i < nIt; ++i) {
        const int slot = i % kSlots;
        if (!wait_bounded(&C.empty[slot], static_cast<uint32_t>((i / kSlots) & 1) ^ 1u, abort_flag)) break;
        unsigned char* dst = base + static_cast<size_t>(slot) * a.slot_bytes;
        if (i < nItA) {
          const int u = i / (f1 - f0), r = f0 + i % (f1 - f0);
          const size_t off = (static_cast<size_t>(C.uexp[u]) * f + r) * d;
          mbar_expect_tx(&C.full[slot], static_cast<uint32_t>(4 * d));
          bulk_load(dst, a.w_gate + off, static_cast<uint32_t>(2 * d), &C.full[slot]);
          bulk_load(dst + 2 * d, a.w_up + off, static_cast<uint32_t>(2 * d), &C.full[slot]);
        } else {
          const int j = i - nItA;
          const int u = j / (n1 - n0), n = n0 + j % (n1 - n0);
          mbar_expect_tx(&C.full[slot], static_cast<uint32_t>(2 * f));
          bulk_load(dst, a.w_down + (static_cast<size_t>(C.uexp[u]) * d + n) * f, static_cast<uint32_t>(2 * f),
                    &C.full[slot]);
        }
      }
      if (i < nIt) abort_cta(C, a.timeouts);
      if (*abort_flag) {
        // copies armed on `full` must land before the CTA goes (bounded)
        for (int s = 0; s < kSlots && s < i; ++s) {
          const int last = s + ((i - 1 - s) / kSlots) * kSlots;
          const uint64_t t1 = globaltimer();
          while (!mbar_try_wait(&C.full[s], static_cast<uint32_t>((last / kSlots) & 1)) &&
                 globaltimer() - t1 < kTimeoutNs) {
          }
        }
      }
    }
  } else {
    // ============================== consumers (warps 1..7) ==============================
    const int cw = warp - 1;
    // phase A: h of the owned f-rows of every chosen expert, for each of its assignments
    for (int i = cw; i < nItA && ok; i += kConsumers) {
      const int slot = i % kSlots;
      ok = __all_sync(0xffffffffu, wait_bounded(&C.full[slot], static_cast<uint32_t>((i / kSlots) & 1), abort_flag));
      if (!ok) break;
      const int u = i / (f1 - f0), r = f0 + i % (f1 - f0);
      const uint16_t* gr = reinterpret_cast<const uint16_t*>(base + static_cast<size_t>(slot) * a.slot_bytes);
      const uint16_t* ur = gr + d;
      for (int q = 0; q < C.una[u]; ++q) {
        const int as = C.ua[u][q], t = as / k;
        const float gv = warp_dot(gr, xs + static_cast<size_t>(t) * d, d, lane);
        const float uv = warp_dot(ur, xs + static_cast<size_t>(t) * d, d, lane);
        if (lane == 0) a.hbuf[static_cast<size_t>(as) * f + r] = gv / (1.f + expf(-gv)) * uv;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[slot]);
    }
    // grid barrier among the consumers: every CTA's h rows are stored
    ok = bar_and(1, kConsumers * 32, ok);
    bool h_armed = false;   // thread 32: the copy of h is in flight on C.hb
    if (threadIdx.x == 32) {
      bool passed = false;
      if (ok) {
        red_release_add(a.gbar, 1u);
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 0;; ++it) {
          if (ld_acquire(a.gbar) >= static_cast<unsigned int>(nC)) {
            passed = true;
            break;
          }
          if ((it & 15) == 15 && (*abort_flag || globaltimer() - t0 > kTimeoutNs)) break;
        }
      }
      if (passed && nu > 0) {
        // h was written through the generic proxy by other CTAs: order it before the bulk copy
        asm volatile("fence.proxy.async.global;" ::: "memory");
        const uint32_t hbytes = static_cast<uint32_t>(nA) * f * 4;
        mbar_expect_tx(&C.hb, hbytes);
        h_armed = true;
        for (uint32_t o = 0; o < hbytes; o += 32768u)
          bulk_load(reinterpret_cast<unsigned char*>(hs) + o, reinterpret_cast<const unsigned char*>(a.hbuf) + o,
                    hbytes - o < 32768u ? hbytes - o : 32768u, &C.hb);
      }
      if (!passed) abort_cta(C, a.timeouts);
    }
    ok = bar_and(1, kConsumers * 32, ok && !*abort_flag);
    if (ok && nu > 0) ok = __all_sync(0xffffffffu, wait_bounded(&C.hb, 0, abort_flag));
    // phase B: the owned d-rows of every chosen expert, for each of its assignments (items i with
    // i % kConsumers == cw, as in phase A)
    for (int i = nItA + ((cw - nItA % kConsumers) + kConsumers) % kConsumers; i < nIt && ok; i += kConsumers) {
      const int j = i - nItA, slot = i % kSlots;
      ok = __all_sync(0xffffffffu, wait_bounded(&C.full[slot], static_cast<uint32_t>((i / kSlots) & 1), abort_flag));
      if (!ok) break;
      const int u = j / (n1 - n0), n = j % (n1 - n0);
      const uint16_t* dr = reinterpret_cast<const uint16_t*>(base + static_cast<size_t>(slot) * a.slot_bytes);
      for (int q = 0; q < C.una[u]; ++q) {
        const int as = C.ua[u][q];
        const float v = warp_dot(dr, hs + static_cast<size_t>(as) * f, f, lane);
        if (lane == 0) C.ypart[as][n] = v;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.empty[slot]);
    }
    ok = bar_and(1, kConsumers * 32, ok);
    if (!ok && lane == 0) abort_cta(C, a.timeouts);
    // y for the owned rows: residual + the chosen experts in slot order
    if (ok) {
      for (int q = threadIdx.x - 32; q < T * (n1 - n0); q += kConsumers * 32) {
        const int t = q / (n1 - n0), n = q % (n1 - n0);
        const size_t o = static_cast<size_t>(t) * d + n0 + n;
        float acc = 0.f;
        for (int i = 0; i < k; ++i) acc = fmaf(C.gsel[t * k + i], C.ypart[t * k + i][n], acc);
        a.y[o] = (a.h_in ? a.h_in[o] : 0.f) + acc;
      }
    }
    if (h_armed && *abort_flag) {
      // the copy of h must land before the CTA goes (bounded)
      const uint64_t t1 = globaltimer();
      while (!mbar_try_wait(&C.hb, 0) && globaltimer() - t1 < kTimeoutNs) {
      }
    }
  }
  // the producer runs on lane 0 alone: its warp meets the CTA barrier converged
  __syncwarp();
  __syncthreads();
}

}  // namespace

bool moe_layer_tiny_supported(int T, int E, int d, int f, int k) {
  if (T < 1 || static_cast<long long>(T) * k > kMaxA || E > kMaxE || d % 8 != 0 || f % 8 != 0) return false;
  const int nC = num_sms();
  if (nC < 1 || (d + nC - 1) / nC > kMaxRowsB) return false;
  const uint32_t slot = static_cast<uint32_t>(4 * d > 2 * f ? 4 * d : 2 * f);
  const TinySmem S = tiny_smem(T, k, d, f, slot);
  // the staging copies (router rows, token rows as f32, gamma) must fit in the ring
  const size_t staging = static_cast<size_t>(E) * d * 2 + static_cast<size_t>(T) * d * 4 + static_cast<size_t>(d) * 4;
  return staging <= S.xs && S.total + 1024 <= static_cast<size_t>(max_smem_optin());
}

size_t moe_layer_tiny_workspace(int T, int f, int k) {
  return 256 + static_cast<size_t>(T) * k * f * 4;
}

zmoe_status moe_layer_tiny(const uint16_t* x, const float* h_in, const float* gamma, float eps, const uint16_t* w_r,
                           const float* logit_bias, const float* sel_bias, const uint16_t* w_gate, const uint16_t* w_up,
                           const uint16_t* w_down, int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                           float* gates, float* margin, uint16_t* x_norm, void* ws, cudaStream_t s) {
  TinyArgs a{};
  a.x_in = x;
  a.h_in = h_in;
  a.gamma = gamma;
  a.eps = eps;
  a.w_r = w_r;
  a.logit_bias = logit_bias;
  a.sel_bias = sel_bias;
  a.w_gate = w_gate;
  a.w_up = w_up;
  a.w_down = w_down;
  a.T = T;
  a.d = d;
  a.f = f;
  a.E = E;
  a.k = k;
  a.y = y;
  a.expert_idx = expert_idx;
  a.gates = gates;
  a.margin = margin;
  a.x_norm = x_norm;
  unsigned char* w = static_cast<unsigned char*>(ws);
  a.gbar = reinterpret_cast<unsigned int*>(w);
  a.hbuf = reinterpret_cast<float*>(w + 256);
  a.timeouts = device_timeout_counter();
  a.slot_bytes = static_cast<uint32_t>(4 * d > 2 * f ? 4 * d : 2 * f);
  const size_t smem = tiny_smem(T, k, d, f, a.slot_bytes).total + 1024;
  if (cudaMemsetAsync(ws, 0, 256, s) != cudaSuccess) return check_launch("zmoe_moe_layer (tiny): clearing the barrier");
  if (cudaFuncSetAttribute(tiny_layer_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return check_launch("zmoe_moe_layer (tiny)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms()));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: they wait on one another once
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, tiny_layer_kernel, a);
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string("zmoe_moe_layer (tiny): ") + cudaGetErrorString(e));
  return check_launch("zmoe_moe_layer (tiny)");
}

}  // namespace zmoe
