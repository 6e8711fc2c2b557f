// Router at prefill sizes on the tensor cores.
//
// The router logits are a dense contraction, logits[T, E] = x[T, d] W_r[E, d]^T (ZONOS2 Technical
// Report digest, "method overview and architecture", items 5-6; the telknet.cc article on ZONOS2,
// section 2.1: a linear router followed by TopK).  On CUDA cores the T E d multiply-adds bound the
// kernel; on tcgen05 they cost nothing next to reading x once from HBM, so this kernel is bound by
// that read (T d 2 bytes).
//
// One CTA per 128 tokens (MMA M = 128, the token rows in TMEM lanes; N = the experts padded to 16 or
// 32 columns, zero rows past E by the copy's fill; K = d in 64-wide stages):
//   warp 0  loads the x box (128 rows x 64 bf16, 16 KB) and the W_r box (EP rows x 64) of each stage
//           with TMA into a ring of kStages;
//   warp 1  allocates TMEM and issues 4 MMAs per stage from one elected lane; tcgen05.commit frees the
//           stage, and a last commit marks the accumulator ready;
//   warps 0-3 then read their 32 TMEM lanes (one token per thread, every logit of it in registers) and
//           take the same selection as the CUDA-core router: q = logits + logit_bias, s = q + sel_bias,
//           top-k of s in ascending expert order with ties to the lower index (a NaN score is never
//           chosen), softmax gates over q (k = 1: p[sel]; k = 2: renormalised over the two), and the
//           selection margin.
// Every wait is bounded: on expiry the CTA counts a device timeout, stops issuing, lets the copies and
// MMAs it issued land, frees TMEM and returns.
#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int kBM = 128;                   // tokens per CTA (MMA M, TMEM lanes)
constexpr int kBK = 64;                    // k per stage (one 128-byte swizzle atom of bf16)
constexpr int kStages = 6;
constexpr int kXBytes = kBM * kBK * 2;     // 16 KB
constexpr int kMaxEP = 32;
constexpr int kWBytesMax = kMaxEP * kBK * 2;   // 4 KB
constexpr int kStageStride = kXBytes + kWBytesMax;
constexpr uint32_t kTmemCols = 32;
constexpr unsigned long long kTimeoutNs = 2000000000ull;

struct __align__(8) RouteCtrl {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t done;
  uint32_t tmem;
  int abort;
  float lb[kMaxEP];
  float sb[kMaxEP];
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kStages) * kStageStride + sizeof(RouteCtrl);

struct RouteArgs {
  const float* logit_bias;
  const float* sel_bias;
  int T, d, E, k;
  int32_t* expert_idx;
  float* gates;
  float* margin;
  unsigned int* timeouts;
};

template <int EP>
__global__ void __launch_bounds__(128, 1) route_tc_kernel(const __grid_constant__ CUtensorMap xmap,
                                                         const __grid_constant__ CUtensorMap wmap,
                                                         const RouteArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  RouteCtrl& C = *reinterpret_cast<RouteCtrl*>(base + static_cast<size_t>(kStages) * kStageStride);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kBM;
  const int nk = (a.d + kBK - 1) / kBK;
  constexpr uint32_t kWBytes = EP * kBK * 2;
  volatile int* abort_flag = &C.abort;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], 1);
    }
    mbar_init(&C.done, 1);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x < EP) {
    const int e = threadIdx.x;
    C.lb[e] = (e < a.E && a.logit_bias) ? a.logit_bias[e] : 0.f;
    C.sb[e] = (e < a.E && a.sel_bias) ? a.sel_bias[e] : 0.f;
  }
  if (warp == 1) tmem_alloc(&C.tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem;

  int issued = 0;   // producer: stages whose copies were issued
  bool ok = true;
  if (warp == 0) {
    // ---------------- producer ----------------
    if (elect_one()) {
      for (int s = 0; s < nk; ++s) {
        const int slot = s % kStages;
        if (s >= kStages && !mbar_wait(&C.empty[slot], static_cast<uint32_t>(((s / kStages) - 1) & 1), abort_flag,
                                       kTimeoutNs)) {
          ok = false;
          break;
        }
        unsigned char* st = base + static_cast<size_t>(slot) * kStageStride;
        mbar_expect_tx(&C.full[slot], static_cast<uint32_t>(kXBytes) + kWBytes);
        tma_load_2d(st, &xmap, &C.full[slot], s * kBK, t0);
        tma_load_2d(st + kXBytes, &wmap, &C.full[slot], s * kBK, 0);
        issued = s + 1;
      }
      if (!ok && atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    constexpr uint32_t idesc = idesc_bf16_f32(kBM, EP);
    int s = 0;
    for (; s < nk; ++s) {
      const int slot = s % kStages;
      const bool got = __all_sync(0xffffffffu, mbar_wait(&C.full[slot], static_cast<uint32_t>((s / kStages) & 1),
                                                         abort_flag, kTimeoutNs));
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (elect_one()) {
        const uint32_t sa = smem_u32(base + static_cast<size_t>(slot) * kStageStride);
        const uint64_t da = sw128_desc(sa), db = sw128_desc(sa + kXBytes);
#pragma unroll
        for (int kk = 0; kk < kBK / 16; ++kk)
          umma_bf16(tmem, da + static_cast<uint64_t>((kk * 32) >> 4), db + static_cast<uint64_t>((kk * 32) >> 4),
                    idesc, (s == 0 && kk == 0) ? 0u : 1u);
        umma_commit(&C.empty[slot]);
      }
      __syncwarp();
    }
    if (!ok && lane == 0 && atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
    // the accumulator is complete (or, after an abort, every issued MMA has finished) when `done` flips
    if (elect_one()) umma_commit(&C.done);
    __syncwarp();
  }

  // ---------------- epilogue: one token per thread ----------------
  // (not cut short by an abort: the MMA warp always commits `done`, and TMEM is freed only after it)
  bool ready = true;
  {
    const uint64_t t1 = globaltimer();
    while (!mbar_try_wait(&C.done, 0u)) {
      if (globaltimer() - t1 > kTimeoutNs) {
        ready = false;
        break;
      }
    }
  }
  tc_fence_after();
  const bool good = __syncthreads_and(ready && !*abort_flag);
  if (good) {
    uint32_t r[kMaxEP];
    const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    if constexpr (EP == 16) {
      tmem_ld16(taddr, *reinterpret_cast<uint32_t (*)[16]>(r));
    } else {
      tmem_ld32(taddr, *reinterpret_cast<uint32_t (*)[32]>(r));
    }
    tmem_wait_ld();
    const int tok = t0 + warp * 32 + lane;
    const int E = a.E, k = a.k;
    float q[EP], sc[EP];
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      q[e] = e < E ? __uint_as_float(r[e]) + C.lb[e] : -INFINITY;
      sc[e] = e < E ? q[e] + C.sb[e] : -INFINITY;
    }
    // ranks 1-3 of s: ascending expert order, a strictly larger score replaces (ties keep the lower index)
    float s1 = -INFINITY, s2 = -INFINITY, s3 = -INFINITY;
    int e1 = -1, e2 = -1;
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      if (e < E && (e1 < 0 ? sc[e] == sc[e] : sc[e] > s1)) {
        s1 = sc[e];
        e1 = e;
      }
    }
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      if (e < E && e != e1 && (e2 < 0 ? sc[e] == sc[e] : sc[e] > s2)) {
        s2 = sc[e];
        e2 = e;
      }
    }
    if (k == 2) {
      int e3 = -1;
#pragma unroll
      for (int e = 0; e < EP; ++e) {
        if (e < E && e != e1 && e != e2 && (e3 < 0 ? sc[e] == sc[e] : sc[e] > s3)) {
          s3 = sc[e];
          e3 = e;
        }
      }
    }
    // softmax over the unbiased q
    float m = -INFINITY;
#pragma unroll
    for (int e = 0; e < EP; ++e)
      if (e < E) m = fmaxf(m, q[e]);
    float z = 0.f, q1 = 0.f, q2 = 0.f;
#pragma unroll
    for (int e = 0; e < EP; ++e) {
      if (e < E) z += expf(q[e] - m);
      if (e == e1) q1 = q[e];
      if (e == e2) q2 = q[e];
    }
    if (tok < a.T) {
      if (k == 1) {
        a.expert_idx[tok] = e1;
        a.gates[tok] = expf(q1 - m) / z;
        if (a.margin) a.margin[tok] = (E > 1) ? s1 - s2 : INFINITY;
      } else {
        const float z1 = expf(q1 - m), z2 = expf(q2 - m);
        const float inv = 1.f / (z1 + z2);
        a.expert_idx[2 * tok] = e1;
        a.expert_idx[2 * tok + 1] = e2;
        a.gates[2 * tok] = z1 * inv;
        a.gates[2 * tok + 1] = z2 * inv;
        if (a.margin) a.margin[tok] = (E > 2) ? fminf(s1 - s2, s2 - s3) : s1 - s2;
      }
    }
  } else if (threadIdx.x == 0) {
    if (atomicExch(&C.abort, 1) == 0) atomicAdd(a.timeouts, 1u);
    // copies issued but never consumed land before the CTA leaves (bounded)
    for (int s = 0; s < issued && s < kStages; ++s) {
      const int last = s + ((issued - 1 - s) / kStages) * kStages;
      const uint64_t t1 = globaltimer();
      while (!mbar_try_wait(&C.full[s % kStages], static_cast<uint32_t>((last / kStages) & 1)) &&
             globaltimer() - t1 < kTimeoutNs) {
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

// Launches the tensor-core router when it applies (bf16, E <= 32, d a multiple of 64, at least
// kRouteTcMinT tokens); returns false, launching nothing, otherwise.
bool launch_route_tc(const void* x, const void* w, const float* lb, const float* sb, int T, int d, int E, int k,
                     int32_t* idx, float* g, float* mg, cudaStream_t s) {
  constexpr int kRouteTcMinT = 2048;
  if (T < kRouteTcMinT || E > kMaxEP || d % kBK != 0) return false;
  const int EP = E <= 16 ? 16 : 32;
  CUtensorMap xm, wm;
  const cuuint64_t xd[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(T)};
  const cuuint64_t wd[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(E)};
  const cuuint64_t st[1] = {static_cast<cuuint64_t>(d) * 2};
  const cuuint32_t xb[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(kBM)};
  const cuuint32_t wb[2] = {static_cast<cuuint32_t>(kBK), static_cast<cuuint32_t>(EP)};
  if (!encode_bf16_map(&xm, x, 2, xd, st, xb) || !encode_bf16_map(&wm, w, 2, wd, st, wb)) return false;
  RouteArgs a{};
  a.logit_bias = lb;
  a.sel_bias = sb;
  a.T = T;
  a.d = d;
  a.E = E;
  a.k = k;
  a.expert_idx = idx;
  a.gates = g;
  a.margin = mg;
  a.timeouts = device_timeout_counter();
  const int grid = (T + kBM - 1) / kBM;
  if (EP == 16) {
    if (cudaFuncSetAttribute(route_tc_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    route_tc_kernel<16><<<grid, 128, kSmemBytes, s>>>(xm, wm, a);
  } else {
    if (cudaFuncSetAttribute(route_tc_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             static_cast<int>(kSmemBytes)) != cudaSuccess) {
      cudaGetLastError();
      return false;
    }
    route_tc_kernel<32><<<grid, 128, kSmemBytes, s>>>(xm, wm, a);
  }
  return true;
}

}  // namespace zmoe
