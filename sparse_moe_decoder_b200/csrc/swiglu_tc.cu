// Grouped SwiGLU on the 5th-generation tensor cores for prefill-size batches, on CTA pairs.
//
// Per expert e over its rows of the permuted activations ("GLU Variants Improve Transformer",
// ZONOS2 Technical Report "Builds on"; SiLU per the telknet.cc article on ZONOS2, section 2.1):
//   gate/up GEMM:  [G | U] = X_e [W_gate,e ; W_up,e]^T,   h = silu(G) * U
//   down GEMM:     y_perm  = h_e W_down,e^T  -> fp32
// h is carried in one of two formats:
//   * f16 (11 significant bits; the down weights are an f16 copy scaled by a power of two per expert,
//     exact for the bf16 weights, zmoe_prepare_w_down_f16): the down GEMM contracts K = f;
//   * a bf16 pair [h_hi | h_lo], h_hi = bf16(h), h_lo = bf16(h - h_hi), with the bf16 down weights:
//     K = 2f over [W_down | W_down].
// Either keeps the rounding of h out of the result's bar (a single bf16 h costs up to 3% of the output
// RMS on skewed gates; f16 costs ~0.3%).
//
// Two CTAs of a cluster share each 256 x 256 tile: tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16),
// issued by the even CTA, reads A rows 0..127 and B rows 0..127 from the even CTA's shared memory and the
// other halves from the odd CTA's, and leaves D rows 0..127 in the even CTA's tensor memory and rows
// 128..255 in the odd CTA's.  Per CTA and 64-wide k-block that is 16 KB of A and 16 KB of B for
// 2 x 128 x 256 x 64 FLOPs, two thirds of the bytes per FLOP of a one-CTA 128 x 256 tile, so a 6-stage
// ring (192 KB) holds more time of MMA work in flight.  Per CTA, 320 threads:
//   warp 0      TMA producer of this CTA's halves (2D tiled loads of the pair, cta_group::2, 128-byte
//               swizzle, no multicast): both CTAs' bytes of a stage complete on the even CTA's stage
//               barrier, which the even producer arms for both;
//   warp 1      even CTA: allocates 512 TMEM columns (two 256-column fp32 accumulators, with the odd
//               CTA), waits for the stage and issues the MMAs from one lane; a commit multicast to both
//               CTAs frees a stage and, per tile, hands the accumulator to both epilogues; odd CTA:
//               allocates with the even CTA.  Barriers that the other CTA's copies or threads complete
//               are polled without suspending the thread (a suspended waiter wakes ~0.5 us late on a
//               remote arrival, which starved the MMAs);
//   warps 2..9  epilogue: tcgen05.ld of this CTA's 128 accumulator rows (a 32-lane quarter and half of
//               the column chunks per warp: two warps per quarter, so the epilogue keeps up with the MMAs),
//               SiLU * up -> h (gate/up) or the scaled fp32 result (down); masked stores of valid rows;
//               then an arrival on the even CTA's accumulator-free barrier.
// Tiles are the flattened (expert, 256-row m-tile, n-tile) space computed on the device from `offsets`,
// dealt round-robin to the CTA pairs; the two accumulators let the epilogue of one tile overlap the main
// loop of the next.  Gate/up tiles take 128 gate rows (even CTA) and the matching 128 up rows (odd CTA)
// of the weights as B, so D's columns 0..127 hold G and 128..255 hold U for 128 features.  Rows of a tile
// past its expert's segment read the next expert's (or zero-filled) rows; they cost MMA work but are never
// stored.
//
// Every wait is bounded (time limit); on expiry the CTA sets its own and its partner's abort flag, counts
// a device timeout, drains its own copies and the MMAs, and both CTAs free their tensor memory together.
#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int BMC = 128;                        // rows of A per CTA (256 per pair)
constexpr int BN = 256;                         // MMA N
constexpr int BNC = 128;                        // rows of B per CTA
constexpr int KB_BYTES = 128;                   // bytes of K per row and stage (one 128-byte swizzle atom)
constexpr int STAGES = 6;
constexpr int A_BYTES = BMC * KB_BYTES;         // 16 KB
constexpr int B_BYTES = BNC * KB_BYTES;         // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 32 KB
constexpr int kThreads = 320;   // warp 0 producer, warp 1 MMA, warps 2..9 epilogue
constexpr int kEpiWarps = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr unsigned long long kTimeoutNs = 2000000000ull;
constexpr int kMaxE = 64;

enum { kGateUp = 0, kDown = 1 };
// Operand formats: bf16 with h as the bf16 pair; bf16 x / gate / up with h and W_down in f16; E4M3 with
// per-row scales (W8A8).
enum { kPair = 0, kF16 = 1, kE4M3 = 2 };

// Elements of K per stage.
__host__ __device__ constexpr int bk_of(int fmt) { return fmt == kE4M3 ? KB_BYTES : KB_BYTES / 2; }

struct TcParams {
  const int32_t* offsets;
  void* out;                 // gate/up: h (f16 [M, f] or bf16 pair [M, 2f]); down: y_perm f32 [M, d]
  const float* down_scale;   // f16 down: [E], multiplies the finished sums; else null
  const float* row_scale;    // E4M3: [M] per-token scale of A's rows (x or h)
  const float* col_scale0;   // E4M3: row scales of the weights: gate [E f] (gate/up) or down [E d]
  const float* col_scale1;   // E4M3 gate/up: up [E f]
  unsigned int* amax;        // E4M3 gate/up: [M] bits of max |f16(h)| per row (atomic max)
  int E, K, out_ld;          // contraction length (A columns); row length of `out`
  int M_total;               // rows of x_perm / h / y_perm: offsets must be a monotone split of [0, M_total]
  int lo_offset;             // bf16 pair: column of h_lo in `out` (= f)
  int kb_wrap;               // B's k-block is kb % kb_wrap (pair down: f / 64; else K / 64)
  int b_rows_per_expert;     // f (gate/up) or d (down)
  int n_tiles;               // n-tiles per m-tile
  unsigned int* timeouts;
  unsigned int* errors;
};

struct __align__(8) Ctrl {
  uint64_t full[STAGES];     // this CTA's bytes of the stage have landed
  uint64_t empty[STAGES];    // the MMAs reading the stage are done (commit multicast to both CTAs)
  uint64_t tfull[2];         // accumulator ready (commit multicast to both CTAs)
  uint64_t tempty[2];        // even CTA: accumulator read by both CTAs' epilogues (8 warp arrivals)
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int off[kMaxE + 1];
  int tile_start[kMaxE + 1];
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + sizeof(Ctrl);

__device__ __forceinline__ void decode_tile(const Ctrl& C, int E, int n_tiles, int t, int& e, int& mt, int& nt) {
  e = 0;
  while (e + 1 < E && C.tile_start[e + 1] <= t) ++e;
  const int local = t - C.tile_start[e];
  mt = local / n_tiles;
  nt = local - mt * n_tiles;
}

// Sets this CTA's abort flag (counting one timeout) and the partner's (not counted there).
__device__ __forceinline__ void set_abort(Ctrl& C, unsigned int* counter, uint32_t peer) {
  if (atomicExch(&C.abort, 1) == 0) {
    if (counter) atomicAdd(counter, 1u);
    const uint32_t remote = mapa_shared(smem_u32(&C.abort), peer);
    asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(1u) : "memory");
  }
}

// silu(g) * u with the fast exponential and division (~2 ulp of fp32, far below the 11 bits of an f16 h or
// the 16 of the bf16 pair): the epilogue computes one per h value, on one warp per SM sub-partition.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.f + __expf(-g)) * u; }

__device__ __forceinline__ uint16_t f32_to_f16_bits(float v) {
  const __half h = __float2half_rn(v);
  return *reinterpret_cast<const uint16_t*>(&h);
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
template <int MODE, int FMT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    tc_ffn_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                  const __grid_constant__ CUtensorMap mapB1, TcParams p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* stages = base;
  Ctrl& C = *reinterpret_cast<Ctrl*>(base + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &C.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const bool even = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&C.full[s], 1);
      mbar_init(&C.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&C.tfull[b], 1);
      mbar_init(&C.tempty[b], 2 * kEpiWarps);   // every epilogue warp of both CTAs
    }
    mbar_init(&C.drain, 1);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (threadIdx.x <= p.E) C.off[threadIdx.x] = p.offsets[threadIdx.x];
  if (warp == 1) tmem_alloc2(&C.tmem_base, TMEM_COLS);
  // both CTAs' barriers are initialised and the columns allocated before either CTA signals the other
  cluster_sync();
  if (threadIdx.x == 0) {
    // offsets that are not a monotone split of [0, M_total] would send rows past the buffers: count a
    // device error and run no tiles
    bool bad = C.off[0] != 0 || C.off[p.E] > p.M_total;
    for (int e = 0; e < p.E; ++e) bad = bad || C.off[e + 1] < C.off[e];
    int acc = 0;
    for (int e = 0; e < p.E; ++e) {
      C.tile_start[e] = acc;
      if (!bad) acc += ((C.off[e + 1] - C.off[e] + 2 * BMC - 1) / (2 * BMC)) * p.n_tiles;
    }
    C.tile_start[p.E] = acc;
    if (bad && even && pair == 0) record_device_error(p.errors);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;
  const int total = C.tile_start[p.E];
  constexpr int BK = bk_of(FMT);
  const int nkb = p.K / BK;

  int issued = 0;   // k-blocks whose loads this CTA's producer issued (producer thread only)
  if (warp == 0) {
    if (lane == 0) {
      // ---------------- TMA producer (this CTA's halves) ----------------
      const CUtensorMap* mB = (MODE == kGateUp && !even) ? &mapB1 : &mapB0;
      int kbt = 0;
      for (int t = pair; t < total && !*abort_flag; t += npairs) {
        int e, mt, nt;
        decode_tile(C, p.E, p.n_tiles, t, e, mt, nt);
        const int arow = C.off[e] + mt * (2 * BMC) + static_cast<int>(rank) * BMC;
        const int brow = MODE == kGateUp ? e * p.b_rows_per_expert + nt * BNC
                                         : e * p.b_rows_per_expert + nt * BN + static_cast<int>(rank) * BNC;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++kbt) {
          const int s = kbt % STAGES;
          const uint32_t ph = static_cast<uint32_t>(kbt / STAGES) & 1u;
          if (!mbar_wait_cluster(&C.empty[s], ph ^ 1u, abort_flag, kTimeoutNs)) {
            set_abort(C, p.timeouts, peer);
            ok = false;
            break;
          }
          // both CTAs' bytes complete on the even CTA's barrier, which the even producer arms for both
          const uint32_t fbar = mapa_shared(smem_u32(&C.full[s]), 0);
          if (even) mbar_expect_tx(&C.full[s], 2 * STAGE_BYTES);
          unsigned char* sa = stages + s * STAGE_BYTES;
          tma_load_2d_pair(sa, &mapA, fbar, kb * BK, arow);
          tma_load_2d_pair(sa + A_BYTES, mB, fbar, (kb % p.kb_wrap) * BK, brow);
        }
        if (!ok) break;
      }
      issued = kbt;
    }
  } else if (warp == 1) {
    if (even) {
      if (lane == 0) {
        // ---------------- MMA issuer (even CTA) ----------------
        constexpr uint32_t idesc = FMT == kE4M3                      ? idesc_e4m3_f32(2 * BMC, BN)
                                   : (MODE == kDown && FMT == kF16) ? idesc_f16_f32(2 * BMC, BN)
                                                                    : idesc_bf16_f32(2 * BMC, BN);
        int kbt = 0, it = 0;
        bool ok = true;
        for (int t = pair; t < total && ok && !*abort_flag; t += npairs, ++it) {
          const int b = it & 1;
          const uint32_t tph = static_cast<uint32_t>(it >> 1) & 1u;
          if (!mbar_wait_cluster(&C.tempty[b], tph ^ 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * BN);
          for (int kb = 0; kb < nkb; ++kb, ++kbt) {
            const int s = kbt % STAGES;
            const uint32_t ph = static_cast<uint32_t>(kbt / STAGES) & 1u;
            if (!mbar_wait_cluster(&C.full[s], ph, abort_flag, kTimeoutNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(stages + s * STAGE_BYTES);
            const uint32_t sb = sa + A_BYTES;
            // four MMAs of 32 bytes of K each (K = 16 bf16 / f16 elements, or 32 E4M3 elements)
#pragma unroll
            for (int kk = 0; kk < KB_BYTES / 32; ++kk) {
              if (FMT == kE4M3)
                umma2_f8(d_tmem, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
              else
                umma2_f16(d_tmem, sw128_desc(sa + kk * 32), sw128_desc(sb + kk * 32), idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            umma2_commit_mc(&C.empty[s], 0x3);
          }
          if (!ok) break;
          umma2_commit_mc(&C.tfull[b], 0x3);
        }
        if (!ok) set_abort(C, p.timeouts, peer);
        // every MMA issued here completes (and its commits have arrived) before the drain barrier flips
        umma2_commit(&C.drain);
        const uint64_t t0 = globaltimer();
        while (!mbar_try_wait(&C.drain, 0) && globaltimer() - t0 < kTimeoutNs) {
        }
      }
    }
  } else {
    // ---------------- epilogue (warps 2..9) ----------------
    // a warp reads the TMEM lanes of its quarter (warp % 4) and one half of each tile's column chunks
    const int quarter = warp & 3;
    const int chalf = (warp - 2) >> 2;
    const uint32_t tempty0 = mapa_shared(smem_u32(&C.tempty[0]), 0);
    const uint32_t tempty1 = mapa_shared(smem_u32(&C.tempty[1]), 0);
    int it = 0;
    for (int t = pair; t < total && !*abort_flag; t += npairs, ++it) {
      const int b = it & 1;
      const uint32_t tph = static_cast<uint32_t>(it >> 1) & 1u;
      if (!mbar_wait(&C.tfull[b], tph, abort_flag, kTimeoutNs)) {
        set_abort(C, p.timeouts, peer);
        break;
      }
      tc_fence_after();
      int e, mt, nt;
      decode_tile(C, p.E, p.n_tiles, t, e, mt, nt);
      const int row = C.off[e] + mt * (2 * BMC) + static_cast<int>(rank) * BMC + quarter * 32 + lane;
      const bool valid = row < C.off[e + 1];
      const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * BN);
      if (MODE == kGateUp) {
        uint16_t* h = static_cast<uint16_t*>(p.out) + static_cast<size_t>(row) * p.out_ld + nt * BNC;
        bool range_ok = true;
        float hmax = 0.f;
        const float rs = (FMT == kE4M3 && valid) ? p.row_scale[row] : 1.f;
        const size_t col0 = static_cast<size_t>(e) * p.b_rows_per_expert + nt * BNC;
#pragma unroll 1
        for (int c = 2 * chalf; c < 2 * chalf + 2; ++c) {
          uint32_t g[32], u[32];
          tmem_ld32(taddr + c * 32, g);
          tmem_ld32(taddr + 128 + c * 32, u);
          tmem_wait_ld();
          if (valid) {
            if (FMT != kPair) {
              // E4M3: the chunk's 32 gate and 32 up weight-row scales, as 16-byte loads (the same for every
              // row of the tile: broadcast from L1)
              float sg[32], su[32];
              if (FMT == kE4M3) {
                const float4* pg = reinterpret_cast<const float4*>(p.col_scale0 + col0 + c * 32);
                const float4* pu = reinterpret_cast<const float4*>(p.col_scale1 + col0 + c * 32);
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                  const float4 a = __ldg(pg + q), b = __ldg(pu + q);
                  sg[4 * q] = a.x; sg[4 * q + 1] = a.y; sg[4 * q + 2] = a.z; sg[4 * q + 3] = a.w;
                  su[4 * q] = b.x; su[4 * q + 1] = b.y; su[4 * q + 2] = b.z; su[4 * q + 3] = b.w;
                }
              }
              uint32_t hv[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                if (FMT == kE4M3) {
                  g0 *= rs * sg[2 * i];
                  g1 *= rs * sg[2 * i + 1];
                  u0 *= rs * su[2 * i];
                  u1 *= rs * su[2 * i + 1];
                }
                const float h0 = silu_mul(g0, u0), h1 = silu_mul(g1, u1);
                range_ok = range_ok && fabsf(h0) < 65504.f && fabsf(h1) < 65504.f;
                const uint16_t b0 = f32_to_f16_bits(h0), b1 = f32_to_f16_bits(h1);
                if (FMT == kE4M3)
                  hmax = fmaxf(hmax, fmaxf(fabsf(__half2float(__ushort_as_half(b0))),
                                           fabsf(__half2float(__ushort_as_half(b1)))));
                hv[i] = static_cast<uint32_t>(b0) | (static_cast<uint32_t>(b1) << 16);
              }
              uint4* dst = reinterpret_cast<uint4*>(h + c * 32);
#pragma unroll
              for (int j = 0; j < 4; ++j) dst[j] = make_uint4(hv[4 * j], hv[4 * j + 1], hv[4 * j + 2], hv[4 * j + 3]);
            } else {
              uint32_t hi[16], lo[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float g0 = __uint_as_float(g[2 * i]), g1 = __uint_as_float(g[2 * i + 1]);
                const float u0 = __uint_as_float(u[2 * i]), u1 = __uint_as_float(u[2 * i + 1]);
                const float h0 = silu_mul(g0, u0), h1 = silu_mul(g1, u1);
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
        }
        // an h beyond f16's range (65504) is a data error: counted, the stored value is +-inf
        if (FMT != kPair && !range_ok) record_device_error(p.errors);
        // the row's largest |h| so far, for its per-token E4M3 scale (non-negative floats order as integers)
        if (FMT == kE4M3 && valid) atomicMax(p.amax + row, __float_as_uint(hmax));
      } else {
        float* y = static_cast<float*>(p.out) + static_cast<size_t>(row) * p.out_ld + nt * BN;
        const float sc = FMT == kF16 ? p.down_scale[e] : ((FMT == kE4M3 && valid) ? p.row_scale[row] : 1.f);
        const float* cs = FMT == kE4M3 ? p.col_scale0 + static_cast<size_t>(e) * p.b_rows_per_expert + nt * BN : nullptr;
#pragma unroll 1
        for (int c = 4 * chalf; c < 4 * chalf + 4; ++c) {
          uint32_t v[32];
          tmem_ld32(taddr + c * 32, v);
          tmem_wait_ld();
          if (valid) {
            float o[32];
            if (FMT == kE4M3) {
              // the chunk's 32 weight-row scales as 16-byte loads
              const float4* pc = reinterpret_cast<const float4*>(cs + c * 32);
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const float4 a = __ldg(pc + q);
                o[4 * q] = __uint_as_float(v[4 * q]) * sc * a.x;
                o[4 * q + 1] = __uint_as_float(v[4 * q + 1]) * sc * a.y;
                o[4 * q + 2] = __uint_as_float(v[4 * q + 2]) * sc * a.z;
                o[4 * q + 3] = __uint_as_float(v[4 * q + 3]) * sc * a.w;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j) o[j] = __uint_as_float(v[j]) * sc;
            }
            float4* dst = reinterpret_cast<float4*>(y + c * 32);
#pragma unroll
            for (int j = 0; j < 8; ++j) dst[j] = make_float4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(b ? tempty1 : tempty0);
    }
  }

  // The producer and MMA roles run on lane 0 alone: the other lanes wait here for it, so that every
  // warp meets the CTA barrier (and warp 1 the TMEM release) converged.
  __syncwarp();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_flag && !even) {
    // After an abort, loads this CTA issued may still be landing in its ring; they complete on the even
    // CTA's barriers, which this CTA cannot wait on: give them a bounded time (far above a load's
    // latency) before the cluster barrier below lets the CTA go.
    const uint64_t t0 = globaltimer();
    while (issued > 0 && globaltimer() - t0 < 200000ull) {
    }
  }
  if (warp == 0 && lane == 0 && *abort_flag && even) {
    // After an abort, loads the MMA warp never consumed may still be landing in this CTA's ring (and the
    // odd CTA's).  The latest phase of stage s belongs to the last k-block issued into it; wait (bounded)
    // until that phase has completed, i.e. until both CTAs' bytes of it have arrived.
    for (int s = 0; s < STAGES; ++s) {
      const int last = issued - 1 - ((issued - 1 - s) % STAGES + STAGES) % STAGES;
      if (last < 0) continue;
      const uint32_t ph = static_cast<uint32_t>(last / STAGES) & 1u;
      const uint64_t t0 = globaltimer();
      while (!mbar_try_wait(&C.full[s], ph) && globaltimer() - t0 < kTimeoutNs) {
      }
    }
  }
  __syncwarp();
  __syncthreads();
  // neither CTA leaves (or frees its columns) while the even CTA's MMAs may read the odd CTA's shared
  // memory or write its tensor memory, or a remote arrival is in flight
  tc_fence_before();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc2(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------

// 2D tensor [outer, inner] of 2-byte elements (row-major), box of box_outer rows x 64 elements, 128-byte
// swizzle.  The copy does not look at the values: bf16 and f16 use the same map.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(KB_BYTES / 2), box_outer};
  return encode_bf16_map(m, ptr, 2, dims, strides, box);
}

// The same for 1-byte elements (E4M3 codes): box of box_outer rows x 128 elements.
bool make_map8(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer) {
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(KB_BYTES), box_outer};
  return encode_map(m, ptr, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, dims, strides, box, CU_TENSOR_MAP_SWIZZLE_128B);
}

// CTA pairs that can be resident at once (clusters of 2 are placed within one GPC), cached per kernel
// and device: the grid is that many pairs, so every pair starts at once and the static tile schedule
// has no second wave.
template <typename K>
int resident_pairs(K kern) {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    cudaGetLastError();
    return num_sms() / 2;
  }
  if (cached[dev] > 0) return cached[dev];
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms() & ~1));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    n = num_sms() / 2;
  }
  cached[dev] = n;
  return n;
}

template <int MODE, int FMT>
zmoe_status launch_tc(const CUtensorMap& a, const CUtensorMap& b0, const CUtensorMap& b1, const TcParams& p,
                      cudaStream_t s) {
  auto kern = tc_ffn_kernel<MODE, FMT>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes)) !=
      cudaSuccess)
    return check_launch("grouped_swiglu (tcgen05): shared memory attribute");
  const int pairs = resident_pairs(kern);
  kern<<<2 * pairs, kThreads, kSmemBytes, s>>>(a, b0, b1, p);
  return check_launch("grouped_swiglu (tcgen05)");
}

TcParams params(const int32_t* offsets, void* out, int E, int K, int out_ld, int M_total, int lo_offset, int kb_wrap,
                int b_rows, int n_tiles) {
  TcParams p{};
  p.offsets = offsets;
  p.out = out;
  p.E = E;
  p.K = K;
  p.out_ld = out_ld;
  p.M_total = M_total;
  p.lo_offset = lo_offset;
  p.kb_wrap = kb_wrap;
  p.b_rows_per_expert = b_rows;
  p.n_tiles = n_tiles;
  p.timeouts = device_timeout_counter();
  p.errors = device_error_counter();
  return p;
}

}  // namespace

bool grouped_swiglu_tc_supported(int d, int f) {
  return d % 256 == 0 && f % 128 == 0 && d >= 256 && f >= 128 && num_sms() >= 2 &&
         kSmemBytes <= static_cast<size_t>(max_smem_optin());
}

size_t grouped_swiglu_tc_workspace(int, int, int, int) { return 0; }

// bf16 down weights: h as the bf16 pair.
zmoe_status grouped_swiglu_tc(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                              const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                              float* y_perm, void*, size_t, cudaStream_t s) {
  if (!grouped_swiglu_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (tcgen05): needs d % 256 == 0, f % 128 == 0, E <= 64");
  CUtensorMap mx, mg, mu, mh, md;
  if (!make_map(&mx, x_perm, d, M_total, BMC) || !make_map(&mg, w_gate, d, static_cast<uint64_t>(E) * f, BNC) ||
      !make_map(&mu, w_up, d, static_cast<uint64_t>(E) * f, BNC) || !make_map(&mh, h, 2 * f, M_total, BMC) ||
      !make_map(&md, w_down, f, static_cast<uint64_t>(E) * d, BNC))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (tcgen05): cuTensorMapEncodeTiled failed");
  constexpr int BK = bk_of(kPair);
  zmoe_status st = launch_tc<kGateUp, kPair>(mx, mg, mu, params(offsets, h, E, d, 2 * f, M_total, f, d / BK, f, f / BNC), s);
  if (st != ZMOE_OK) return st;
  return launch_tc<kDown, kPair>(mh, md, md, params(offsets, y_perm, E, 2 * f, d, M_total, 0, f / BK, d, d / BN), s);
}

// f16 down weights (prepared, with per-expert scales): h in f16.
zmoe_status grouped_swiglu_tc_f16h(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                                   const uint16_t* w_up, const uint16_t* w_down_f16, const float* down_scale, int E,
                                   int d, int f, uint16_t* h, float* y_perm, cudaStream_t s) {
  if (!grouped_swiglu_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (tcgen05): needs d % 256 == 0, f % 128 == 0, E <= 64");
  CUtensorMap mx, mg, mu, mh, md;
  if (!make_map(&mx, x_perm, d, M_total, BMC) || !make_map(&mg, w_gate, d, static_cast<uint64_t>(E) * f, BNC) ||
      !make_map(&mu, w_up, d, static_cast<uint64_t>(E) * f, BNC) || !make_map(&mh, h, f, M_total, BMC) ||
      !make_map(&md, w_down_f16, f, static_cast<uint64_t>(E) * d, BNC))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (tcgen05): cuTensorMapEncodeTiled failed");
  constexpr int BK = bk_of(kF16);
  zmoe_status st = launch_tc<kGateUp, kF16>(mx, mg, mu, params(offsets, h, E, d, f, M_total, 0, d / BK, f, f / BNC), s);
  if (st != ZMOE_OK) return st;
  TcParams dn = params(offsets, y_perm, E, f, d, M_total, 0, f / BK, d, d / BN);
  dn.down_scale = down_scale;
  return launch_tc<kDown, kF16>(mh, md, md, dn, s);
}

// W8A8: the gate/up GEMM on E4M3 x rows (per-token scales sx) and E4M3 weights (row scales); writes h in
// f16 and each row's max |h| (amax, zeroed by the caller).
zmoe_status grouped_gateup_tc_e4m3(const uint8_t* xq, const float* sx, const int32_t* offsets, int M_total,
                                   const uint8_t* q_gate, const float* s_gate, const uint8_t* q_up, const float* s_up,
                                   int E, int d, int f, uint16_t* h16, unsigned int* amax, cudaStream_t s) {
  if (!grouped_swiglu_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (fp8): needs d % 256 == 0, f % 128 == 0, E <= 64");
  CUtensorMap mx, mg, mu;
  if (!make_map8(&mx, xq, d, M_total, BMC) || !make_map8(&mg, q_gate, d, static_cast<uint64_t>(E) * f, BNC) ||
      !make_map8(&mu, q_up, d, static_cast<uint64_t>(E) * f, BNC))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (fp8): cuTensorMapEncodeTiled failed");
  constexpr int BK = bk_of(kE4M3);
  TcParams gu = params(offsets, h16, E, d, f, M_total, 0, d / BK, f, f / BNC);
  gu.row_scale = sx;
  gu.col_scale0 = s_gate;
  gu.col_scale1 = s_up;
  gu.amax = amax;
  return launch_tc<kGateUp, kE4M3>(mx, mg, mu, gu, s);
}

// W8A8: the down GEMM on E4M3 h rows (per-token scales sh) and E4M3 W_down (row scales) -> y_perm f32.
zmoe_status grouped_down_tc_e4m3(const uint8_t* hq, const float* sh, const int32_t* offsets, int M_total,
                                 const uint8_t* q_down, const float* s_down, int E, int d, int f, float* y_perm,
                                 cudaStream_t s) {
  if (!grouped_swiglu_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (fp8): needs d % 256 == 0, f % 128 == 0, E <= 64");
  CUtensorMap mh, md;
  if (!make_map8(&mh, hq, f, M_total, BMC) || !make_map8(&md, q_down, f, static_cast<uint64_t>(E) * d, BNC))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (fp8): cuTensorMapEncodeTiled failed");
  constexpr int BK = bk_of(kE4M3);
  TcParams dn = params(offsets, y_perm, E, f, d, M_total, 0, f / BK, d, d / BN);
  dn.row_scale = sh;
  dn.col_scale0 = s_down;
  return launch_tc<kDown, kE4M3>(mh, md, md, dn, s);
}

}  // namespace zmoe
