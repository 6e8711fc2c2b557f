// Grouped SwiGLU on the 5th-generation tensor cores for prefill-size batches.
//
// Per expert e over its rows of the permuted activations ("GLU Variants Improve Transformer",
// ZONOS2 Technical Report "Builds on"; SiLU per the telknet.cc article on ZONOS2, section 2.1):
//   gate/up GEMM:  [G | U] = X_e [W_gate,e ; W_up,e]^T,   h = silu(G) * U
//                  h is stored as a bf16 pair [h_hi | h_lo], h_hi = bf16(h), h_lo = bf16(h - h_hi)
//   down GEMM:     y_perm  = [h_hi | h_lo]_e [W_down,e | W_down,e]^T   (K = 2f)  -> fp32
// Carrying h to ~16 significant bits keeps the bf16 rounding of h out of the result (a single
// bf16 h costs up to 3% of the output RMS on skewed gates); both MMA operands stay bf16.
//
// One persistent CTA per SM, 192 threads in three roles:
//   warp 0      TMA producer: 2D tiled bulk-tensor loads (128-byte swizzle, no multicast) of a
//               128 x 64 A tile and a 256 x 64 B tile per stage into a 4-stage shared ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 fp32 accumulators) and, from one lane,
//               issues tcgen05.mma.cta_group::1.kind::f16 (M = 128, N = 256, K = 16, bf16 in, fp32
//               accumulate); tcgen05.commit releases a stage, and the finished accumulator;
//   warps 2..5  epilogue: tcgen05.ld of their 32-lane quarter of the accumulator, the SiLU * up
//               product (gate/up) or the fp32 result (down), masked stores of valid rows.
// Tiles are the flattened (expert, m-tile, n-tile) space computed on the device from `offsets`
// (no host round trip), dealt round-robin to the CTAs; the two accumulators let the epilogue of
// one tile overlap the main loop of the next.  Gate/up tiles put 128 gate rows and the matching
// 128 up rows of the weights side by side in N, so one accumulator row holds both operands of
// SiLU * up for 128 features.  A tile's rows past its expert's segment read the next expert's
// (or zero-filled) rows; they cost MMA work but are never stored.
//
// Every mbarrier wait is bounded (time limit); on expiry the CTA sets an abort flag, counts a
// device timeout, drains its own copies and MMAs, frees its TMEM and returns.
#include <cuda.h>   // CUtensorMap and its enums (the encoder is fetched from the driver at run time)

#include <mutex>

#include "common.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int kThreads = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr unsigned long long kTimeoutNs = 2000000000ull;   // 2 s
constexpr int kMaxE = 64;

enum { kGateUp = 0, kDown = 1 };

struct TcParams {
  const int32_t* offsets;
  void* out;                 // gate/up: h bf16 [M, f]; down: y_perm f32 [M, d]
  int E, K, out_ld;          // contraction length (A columns); row length of `out`
  int lo_offset;             // gate/up: column of h_lo in `out` (= f)
  int kb_wrap;               // B's k-block index is kb % kb_wrap (down: f / 64; gate/up: K / 64)
  int b_rows_per_expert;     // f (gate/up) or d (down)
  int n_tiles;               // n-tiles per m-tile
  unsigned int* timeouts;
};

struct __align__(8) Ctrl {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int off[kMaxE + 1];
  int tile_start[kMaxE + 1];
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + sizeof(Ctrl);

// ------------------------------------------------------------------------------------------
// PTX wrappers
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Waits for the phase of parity `parity` of `bar` to complete.  Returns false when the CTA
// was aborted or the time limit passed (the caller then sets the abort flag).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0) {
      if (*abort) return false;
      if (globaltimer() - t0 > kTimeoutNs) return false;
    }
  }
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Shared-memory matrix descriptor: K-major operand in 128-byte swizzle atoms (8 rows x 128 B,
// stacked every 1024 B along M/N), sm_100 descriptor version 1.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);    // start address, 16-byte units
  d |= static_cast<uint64_t>(1) << 16;                    // leading byte offset (unused when swizzled)
  d |= static_cast<uint64_t>(1024 >> 4) << 32;            // stride byte offset: next 8-row group
  d |= static_cast<uint64_t>(1) << 46;                    // descriptor version
  d |= static_cast<uint64_t>(2) << 61;                    // SWIZZLE_128B
  return d;
}

// Instruction descriptor of kind::f16: bf16 A and B (K-major), fp32 accumulator, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(N >> 3) << 17)     // N / 8
         | (static_cast<uint32_t>(M >> 4) << 24);    // M / 16
}

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate));
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void decode_tile(const Ctrl& C, int E, int n_tiles, int t, int& e, int& mt, int& nt) {
  e = 0;
  while (e + 1 < E && C.tile_start[e + 1] <= t) ++e;
  const int local = t - C.tile_start[e];
  mt = local / n_tiles;
  nt = local - mt * n_tiles;
}

__device__ __forceinline__ void set_abort(Ctrl& C, unsigned int* counter) {
  if (atomicExch(&C.abort, 1) == 0 && counter) atomicAdd(counter, 1u);
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    tc_ffn_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                  const __grid_constant__ CUtensorMap mapB1, TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stages = base;
  Ctrl& C = *reinterpret_cast<Ctrl*>(base + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &C.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&C.tfull[b], 1);
      mbar_init(&C.tempty[b], 4);
    }
    mbar_init(&C.drain, 1);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (threadIdx.x <= p.E) C.off[threadIdx.x] = p.offsets[threadIdx.x];
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&C.tmem_base)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int e = 0; e < p.E; ++e) {
      C.tile_start[e] = acc;
      acc += ((C.off[e + 1] - C.off[e] + BM - 1) / BM) * p.n_tiles;
    }
    C.tile_start[p.E] = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;
  const int total = C.tile_start[p.E];
  const int nkb = p.K / BK;
  constexpr int B_HALF = B_BYTES / 2;

  int issued = 0;   // k-blocks whose loads the producer issued (producer thread only)
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int kbt = 0;
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x) {
        int e, mt, nt;
        decode_tile(C, p.E, p.n_tiles, t, e, mt, nt);
        const int arow = C.off[e] + mt * BM;
        const int brow = e * p.b_rows_per_expert + nt * (MODE == kGateUp ? 128 : 256);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kbt) {
          const int s = kbt % STAGES;
          const uint32_t ph = static_cast<uint32_t>(kbt / STAGES) & 1u;
          if (!mbar_wait(&C.empty[s], ph ^ 1u, abort_flag)) {
            set_abort(C, p.timeouts);
            ok = false;
            break;
          }
          mbar_expect_tx(&C.full[s], STAGE_BYTES);
          unsigned char* sa = stages + s * STAGE_BYTES;
          unsigned char* sb = sa + A_BYTES;
          const int kbb = (kb % p.kb_wrap) * BK;
          tma_load_2d(sa, &mapA, &C.full[s], kb * BK, arow);
          if (MODE == kGateUp) {
            tma_load_2d(sb, &mapB0, &C.full[s], kbb, brow);
            tma_load_2d(sb + B_HALF, &mapB1, &C.full[s], kbb, brow);
          } else {
            tma_load_2d(sb, &mapB0, &C.full[s], kbb, brow);
            tma_load_2d(sb + B_HALF, &mapB0, &C.full[s], kbb, brow + 128);
          }
        }
        if (!ok) break;
      }
      issued = kbt;
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
      int kbt = 0, it = 0;
      for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++it) {
        const int b = it & 1;
        const uint32_t tph = static_cast<uint32_t>(it >> 1) & 1u;
        if (!mbar_wait(&C.tempty[b], tph ^ 1u, abort_flag)) {
          set_abort(C, p.timeouts);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * BN);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kbt) {
          const int s = kbt % STAGES;
          const uint32_t ph = static_cast<uint32_t>(kbt / STAGES) & 1u;
          if (!mbar_wait(&C.full[s], ph, abort_flag)) {
            set_abort(C, p.timeouts);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(stages + s * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            umma_bf16(d_tmem, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
          umma_commit(&C.empty[s]);
        }
        if (!ok) break;
        umma_commit(&C.tfull[b]);
      }
      // all MMAs issued by this thread complete before the drain barrier flips
      umma_commit(&C.drain);
      if (!mbar_wait(&C.drain, 0, abort_flag)) {
        // aborted: wait once more without the abort short-cut, bounded by the time limit
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&C.drain, 0) && globaltimer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..5) ----------------
    const int quarter = warp & 3;
    int it = 0;
    for (int t = blockIdx.x; t < total && !*abort_flag; t += gridDim.x, ++it) {
      const int b = it & 1;
      const uint32_t tph = static_cast<uint32_t>(it >> 1) & 1u;
      if (!mbar_wait(&C.tfull[b], tph, abort_flag)) {
        set_abort(C, p.timeouts);
        break;
      }
      tc_fence_after();
      int e, mt, nt;
      decode_tile(C, p.E, p.n_tiles, t, e, mt, nt);
      const int row = C.off[e] + mt * BM + quarter * 32 + lane;
      const bool valid = row < C.off[e + 1];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * BN);
      if (MODE == kGateUp) {
        uint16_t* h = static_cast<uint16_t*>(p.out) + static_cast<size_t>(row) * p.out_ld + nt * 128;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(taddr + c * 32, g);
          tmem_ld32(taddr + 128 + c * 32, u);
          tmem_wait_ld();
          if (valid) {
            uint32_t hi[16], lo[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
              const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
              const float h0 = g0 / (1.f + expf(-g0)) * u0, h1 = g1 / (1.f + expf(-g1)) * u1;
              hi[i] = pack_bf16x2(h0, h1);
              lo[i] = pack_bf16x2(h0 - __uint_as_float(hi[i] << 16), h1 - __uint_as_float(hi[i] & 0xFFFF0000u));
            }
            uint4* dst = reinterpret_cast<uint4*>(h + c * 32);
            uint4* dlo = reinterpret_cast<uint4*>(h + p.lo_offset + c * 32);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              dst[j] = make_uint4(hi[4 * j], hi[4 * j + 1], hi[4 * j + 2], hi[4 * j + 3]);
              dlo[j] = make_uint4(lo[4 * j], lo[4 * j + 1], lo[4 * j + 2], lo[4 * j + 3]);
            }
          }
        }
      } else {
        float* y = static_cast<float*>(p.out) + static_cast<size_t>(row) * p.out_ld + nt * 256;
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          if (valid) {
            float4* dst = reinterpret_cast<float4*>(y + c * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j)
              dst[j] = make_float4(__uint_as_float(v[4 * j]), __uint_as_float(v[4 * j + 1]),
                                   __uint_as_float(v[4 * j + 2]), __uint_as_float(v[4 * j + 3]));
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&C.tempty[b]);
    }
  }

  // The producer and MMA roles run on lane 0 alone: the other lanes wait here for it, so that every
  // warp meets the CTA barrier (and warp 1 the TMEM release) converged.
  __syncwarp();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag) {
    // After an abort, loads the MMA warp never consumed may still be landing in the ring.  The
    // latest phase of stage s belongs to the last k-block issued into it; wait (bounded) until
    // that phase has completed, i.e. until its bytes have arrived.
    for (int s = 0; s < STAGES; ++s) {
      const int last = issued - 1 - ((issued - 1 - s) % STAGES + STAGES) % STAGES;
      if (last < 0) continue;
      const uint32_t ph = static_cast<uint32_t>(last / STAGES) & 1u;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&C.full[s], ph) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2D bf16 tensor [outer, inner] (row-major), box of box_outer rows x 64 elements, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(BK), box_outer};
  const cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
zmoe_status launch_tc(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const TcParams& p,
                      cudaStream_t s) {
  auto kern = tc_ffn_kernel<MODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes)) !=
      cudaSuccess)
    return check_launch("grouped_swiglu (tcgen05): shared memory attribute");
  kern<<<num_sms(), kThreads, kSmemBytes, s>>>(a, b0, b1, p);
  return check_launch("grouped_swiglu (tcgen05)");
}

}  // namespace

bool grouped_swiglu_tc_supported(int d, int f) {
  return d % 256 == 0 && f % 128 == 0 && d >= 256 && f >= 128 && kSmemBytes <= static_cast<size_t>(max_smem_optin());
}

size_t grouped_swiglu_tc_workspace(int, int, int, int) { return 0; }

zmoe_status grouped_swiglu_tc(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                              const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                              float* y_perm, void*, size_t, cudaStream_t s) {
  if (!grouped_swiglu_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (tcgen05): needs d % 256 == 0, f % 128 == 0, E <= 64");
  CUtensorMap mx, mg, mu, mh, md;
  if (!make_map(&mx, x_perm, d, M_total, BM) || !make_map(&mg, w_gate, d, static_cast<uint64_t>(E) * f, 128) ||
      !make_map(&mu, w_up, d, static_cast<uint64_t>(E) * f, 128) || !make_map(&mh, h, 2 * f, M_total, BM) ||
      !make_map(&md, w_down, f, static_cast<uint64_t>(E) * d, 128))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (tcgen05): cuTensorMapEncodeTiled failed");
  unsigned int* tmo = device_timeout_counter();
  TcParams gu{offsets, h, E, d, 2 * f, f, d / BK, f, f / 128, tmo};
  zmoe_status st = launch_tc<kGateUp>(mx, mg, mu, gu, s);
  if (st != ZMOE_OK) return st;
  TcParams dn{offsets, y_perm, E, 2 * f, d, 0, f / BK, d, d / 256, tmo};
  return launch_tc<kDown>(mh, md, md, dn, s);
}

}  // namespace zmoe
