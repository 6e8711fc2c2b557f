// Grouped SwiGLU for decode-size batches: one persistent launch that streams the touched
// experts' weights from HBM at full rate (HBM-bound).
//
// Per expert e over its rows of the permuted activations ("GLU Variants Improve Transformer",
// ZONOS2 Technical Report "Builds on"; SiLU per the telknet.cc article on ZONOS2, section 2.1):
//   phase A (gate/up): h = silu(x W_gate[e]^T) * (x W_up[e]^T), stored as the bf16 pair
//                      h_hi = bf16(h), h_lo = bf16(h - h_hi)
//   phase B (down):    y_perm = h_hi W_down[e]^T + h_lo W_down[e]^T          (fp32)
//
// With a few rows per expert there are ~8 FLOP per weight byte, so the time is the time to
// stream the weights once.  Design:
//   * One CTA per SM (cooperative launch: all CTAs are resident), one producer warp and kCons = 4
//     consumer warps.  Each CTA takes an equal, contiguous share of the phase-A unit list and of
//     the phase-B unit list (a unit is 16 output features: 16 gate + 16 up rows, or 16 rows of
//     W_down), computed on the device from `offsets`.
//   * Weights move in 32 KB stages, each ONE 3D TMA box (16 rows x 1024 k, landing as
//     [k-chunk][row][128 B] with 128-byte swizzle).  TMA throughput per SM is bound by boxes per
//     second, so one large box per stage is what reaches full HBM rate (measured on this part:
//     8 KB boxes ~2.7 TB/s, 16 KB ~5.3 TB/s, 32 KB ~6.7-6.8 TB/s, whether a box walks rows or
//     k-chunks first).
//   * Every consumer warp owns one stage slot, so a slot's successive phases always belong to the
//     same warp (no parity aliasing); the producer thread polls all slots (mbarrier.test_wait,
//     never suspending) and refills whichever frees first, and loads each block's token rows (x
//     rows, or h-pair rows, landing as [k-chunk][row][128 B]) once the consumers ask for them.
//   * Consumers: swap-AB mma.sync (weight rows = M 16, tokens = N 8, bf16 in, fp32 accumulate)
//     straight from the swizzled buffers.  In every buffer a line's swizzle key is its row mod 8;
//     MMA row g (and token g) is taken from buffer row rho(g) = g / 2 + 4 (g % 2), so the two rows
//     of a quarter-warp have keys differing in bit 2 and its 16-byte fragment reads hit 8 distinct
//     bank groups with two plain loads.  The epilogue maps rows and columns back through rho.
//     The four MMAs of a chunk accumulate into four registers sets (independent chains).  Only
//     the token groups that hold rows are multiplied.
//   * Gate and up stages of a unit accumulate into two register sets whose lanes hold the same
//     (feature, token) pairs, so silu(gate) * up is formed in registers; h is stored as the pair
//     h_hi = bf16(h), h_lo = bf16(h - h_hi).  In phase B each W_down fragment multiplies both the
//     h_hi and the h_lo rows.
//   * After a block's phase-A units, each warp release-adds its unit count to ready[e] (one fence
//     per warp per block).  Before a phase-B block of expert e, consumer warp 0 acquire-loads
//     ready[e] until all of e's phase-A units are done; the consumers then request the block's
//     tile and the producer fences the async proxy and loads the h rows.  The W_down stages do
//     not depend on h, so they keep streaming while the last gate/up units drain.
//   * Every wait is bounded (time limit): on expiry the CTA counts a device timeout, aborts,
//     drains its own copies in flight and returns.
#include <cuda.h>

#include "common.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

constexpr int kCons = 4;                      // consumer warps, one stage slot each
constexpr int kThreads = (kCons + 1) * 32;    // + producer warp
constexpr int kStageRows = 16;                // weight rows per stage (the MMA's M)
constexpr int kMaxStageChunks = 16;           // 64-wide k chunks per stage (1024 k)
constexpr int kStageBytes = kStageRows * kMaxStageChunks * 128;   // 32 KB
constexpr int kTokA = 24;                     // token rows per phase-A block (3 groups of 8)
constexpr int kTokB = 8;                      // token rows per phase-B block (1 group)
constexpr int kXTileBytes = 98304;            // max(kTokA * d * 2, kTokB * 2f * 2) at d 2048, f 3072
constexpr int kMaxE = 64;
constexpr unsigned long long kTimeoutNs = 2000000000ull;

struct DecodeArgs {
  const int32_t* offsets;   // [E + 1]
  uint16_t* h;              // [M, 2f]  h_hi | h_lo
  float* y;                 // [M, d]
  unsigned int* ready;      // [E] completed phase-A units per expert (zero at launch)
  unsigned int* timeouts;
  int E, d, f;
  int xa_box;               // 64-wide chunks per phase-A token-tile load (divides d / 64)
  int sc_a, sc_b;           // 64-wide chunks per weight stage in phase A (of d) / phase B (of f)
};

struct __align__(8) Ctrl {
  uint64_t full[kCons];     // slot of consumer warp w holds its next stage
  uint64_t empty[kCons];    // consumer warp w released its slot
  uint64_t x_full;   // the token tile of block b has landed (phase b)
  uint64_t x_req;    // every consumer warp is ready for block b's tile (phase b)
  int abort;
  int nseg_a, nseg_b;
  int off[kMaxE + 1];
  int seg_a[kMaxE + 1];     // first phase-A segment (token block) of each expert
  int seg_b[kMaxE + 1];
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(kCons) * kStageBytes + kXTileBytes + sizeof(Ctrl);

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

// Non-blocking test of the same condition (never suspends the thread).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait; false when the CTA was aborted or the time limit passed.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 63) == 0 && (*abort || globaltimer() - t0 > kTimeoutNs)) return false;
  }
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

__device__ __forceinline__ unsigned int ld_acquire(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.global.acquire.gpu.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void red_release_add(unsigned int* p, unsigned int v) {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
  asm volatile("red.relaxed.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Loads the two 16-byte halves (k = q*8.. into v0, k = 32 + q*8.. into v1) of one 64-wide chunk
// held in a 128-byte line whose swizzle key (line index mod 8) is `key`.
__device__ __forceinline__ void ld_line(uint32_t line, int key, int q, uint4& v0, uint4& v1) {
  const uint32_t a = line + static_cast<uint32_t>((q ^ key) << 4);
  const uint32_t b = line + static_cast<uint32_t>(((4 + q) ^ key) << 4);
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v0.x), "=r"(v0.y), "=r"(v0.z), "=r"(v0.w) : "r"(a));
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v1.x), "=r"(v1.y), "=r"(v1.z), "=r"(v1.w) : "r"(b));
}

// The four MMAs of one 64-wide chunk: A rows g (lo0 / lo1) and g + 8 (hi0 / hi1), B token
// fragments b0 (k = q*8..) and b1 (k = 32 + q*8..); the same k permutation on both sides.
__device__ __forceinline__ void mma_chunk(float (&c)[4], const uint4& lo0, const uint4& lo1, const uint4& hi0,
                                          const uint4& hi1, const uint4& b0, const uint4& b1) {
  mma16816(c, lo0.x, hi0.x, lo0.y, hi0.y, b0.x, b0.y);
  mma16816(c, lo0.z, hi0.z, lo0.w, hi0.w, b0.z, b0.w);
  mma16816(c, lo1.x, hi1.x, lo1.y, hi1.y, b1.x, b1.y);
  mma16816(c, lo1.z, hi1.z, lo1.w, hi1.w, b1.z, b1.w);
}

// The same four MMAs, each into its own accumulator: four independent dependency chains.
__device__ __forceinline__ void mma_chunk4(float (&c)[4][4], const uint4& lo0, const uint4& lo1, const uint4& hi0,
                                           const uint4& hi1, const uint4& b0, const uint4& b1) {
  mma16816(c[0], lo0.x, hi0.x, lo0.y, hi0.y, b0.x, b0.y);
  mma16816(c[1], lo0.z, hi0.z, lo0.w, hi0.w, b0.z, b0.w);
  mma16816(c[2], lo1.x, hi1.x, lo1.y, hi1.y, b1.x, b1.y);
  mma16816(c[3], lo1.z, hi1.z, lo1.w, hi1.w, b1.z, b1.w);
}

// ------------------------------------------------------------------------------------------
// work decomposition (identical in every role)
// ------------------------------------------------------------------------------------------
// A "block" is a run of consecutive units of this CTA that share one token block (one x tile).
struct Block {
  int phase;       // 0: gate/up, 1: down
  int e;           // expert
  int row0, rows;  // first permuted row of the token block, rows in it
  int u0, n;       // first unit (within the phase) and number of units of this CTA in the block
  int nb0;         // row-block index of the first unit
};

struct Plan {
  int a_begin, a_end, b_begin, b_end;   // this CTA's unit ranges
  int nblk_a, nblk_b;                   // units per token block
};

__device__ __forceinline__ void locate_seg(const int* seg, const int* off, int E, int tok, int s, int& e, int& row0,
                                           int& rows) {
  e = 0;
  while (e + 1 < E && seg[e + 1] <= s) ++e;
  row0 = off[e] + (s - seg[e]) * tok;
  const int left = off[e + 1] - row0;
  rows = left < tok ? left : tok;
}

// The block that starts at unit u of the given phase (u within this CTA's range).
__device__ __forceinline__ Block make_block(const Ctrl& C, const Plan& P, int E, int phase, int u) {
  Block b;
  b.phase = phase;
  const int nblk = phase ? P.nblk_b : P.nblk_a;
  const int end = phase ? P.b_end : P.a_end;
  const int s = u / nblk;
  locate_seg(phase ? C.seg_b : C.seg_a, C.off, E, phase ? kTokB : kTokA, s, b.e, b.row0, b.rows);
  b.u0 = u;
  b.nb0 = u - s * nblk;
  const int seg_end = (s + 1) * nblk;
  b.n = (seg_end < end ? seg_end : end) - u;
  return b;
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    decode_ffn_kernel(const __grid_constant__ CUtensorMap mapWg, const __grid_constant__ CUtensorMap mapWu,
                      const __grid_constant__ CUtensorMap mapWd, const __grid_constant__ CUtensorMap mapX,
                      const __grid_constant__ CUtensorMap mapH, DecodeArgs p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* ring = base;                                   // [kCons][kStageBytes]
  unsigned char* xtile = base + kCons * kStageBytes;            // [kXTileBytes]
  Ctrl& C = *reinterpret_cast<Ctrl*>(xtile + kXTileBytes);
  volatile int* abort_flag = &C.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;

  if (threadIdx.x == 0) {
    for (int w = 0; w < kCons; ++w) {
      mbar_init(&C.full[w], 1);
      mbar_init(&C.empty[w], 1);
    }
    mbar_init(&C.x_full, 1);
    mbar_init(&C.x_req, kCons);
    C.abort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int i = threadIdx.x; i <= E; i += blockDim.x) C.off[i] = p.offsets[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int a = 0, b = 0;
    for (int e = 0; e < E; ++e) {
      const int m = C.off[e + 1] - C.off[e];
      C.seg_a[e] = a;
      C.seg_b[e] = b;
      a += (m + kTokA - 1) / kTokA;
      b += (m + kTokB - 1) / kTokB;
    }
    C.seg_a[E] = a;
    C.seg_b[E] = b;
    C.nseg_a = a;
    C.nseg_b = b;
  }
  __syncthreads();

  Plan P;
  P.nblk_a = p.f / kStageRows;      // phase-A unit: 16 features (16 gate + 16 up rows)
  P.nblk_b = p.d / kStageRows;      // phase-B unit: 16 rows of W_down
  {
    const long long UA = static_cast<long long>(C.nseg_a) * P.nblk_a;
    const long long UB = static_cast<long long>(C.nseg_b) * P.nblk_b;
    P.a_begin = static_cast<int>(UA * blockIdx.x / gridDim.x);
    P.a_end = static_cast<int>(UA * (blockIdx.x + 1) / gridDim.x);
    P.b_begin = static_cast<int>(UB * blockIdx.x / gridDim.x);
    P.b_end = static_cast<int>(UB * (blockIdx.x + 1) / gridDim.x);
  }
  // stages per unit: phase A alternates gate / up stages over d / (64 sc_a) k-parts
  const int nks_a = 2 * (p.d / (64 * p.sc_a));
  const int nks_b = p.f / (64 * p.sc_b);

  if (warp == kCons) {
    // ===================================== producer =====================================
    if (lane == 0) {
      int issued[kCons];
#pragma unroll
      for (int w = 0; w < kCons; ++w) issued[w] = 0;
      int blk = 0;
      bool ok = true;
      for (int phase = 0; phase < 2 && ok; ++phase) {
        const int u_end = phase ? P.b_end : P.a_end;
        const int nks = phase ? nks_b : nks_a;
        const int sc = phase ? p.sc_b : p.sc_a;
        const uint32_t stage_bytes = static_cast<uint32_t>(sc * kStageRows * 128);
        for (int u = phase ? P.b_begin : P.a_begin; u < u_end && ok; ++blk) {
          const Block B = make_block(C, P, E, phase, u);
          // warp w works on units w, w + kCons, ... of the block, nks stages each
          int left[kCons], cur_i[kCons], cur_ks[kCons];
          int total = 0;
#pragma unroll
          for (int w = 0; w < kCons; ++w) {
            left[w] = (B.n > w) ? ((B.n - w + kCons - 1) / kCons) * nks : 0;
            cur_i[w] = w;
            cur_ks[w] = 0;
            total += left[w];
          }
          bool x_pending = true;
          const uint64_t t0 = globaltimer();
          for (uint32_t it = 0; ok && (total > 0 || x_pending); ++it) {
            // this block's token tile, once every consumer warp has asked for it
            if (x_pending && mbar_test(&C.x_req, static_cast<uint32_t>(blk & 1))) {
              if (phase) {
                asm volatile("fence.proxy.async.global;" ::: "memory");
                mbar_expect_tx(&C.x_full, static_cast<uint32_t>(kTokB * 2 * p.f * 2));
                tma_load_3d(xtile, &mapH, &C.x_full, 0, B.row0, 0);
              } else {
                const int nch = p.d / 64;
                mbar_expect_tx(&C.x_full, static_cast<uint32_t>(kTokA * p.d * 2));
                for (int c = 0; c < nch; c += p.xa_box)
                  tma_load_3d(xtile + c * kTokA * 128, &mapX, &C.x_full, 0, B.row0, c);
              }
              x_pending = false;
            }
            // refill every free slot with its warp's next stage
#pragma unroll
            for (int w = 0; w < kCons; ++w) {
              if (left[w] > 0 && mbar_test(&C.empty[w], static_cast<uint32_t>(issued[w] & 1) ^ 1u)) {
                const int nb = B.nb0 + cur_i[w];
                const int ks = cur_ks[w];
                unsigned char* dst = ring + w * kStageBytes;
                mbar_expect_tx(&C.full[w], stage_bytes);
                if (phase) {
                  tma_load_3d(dst, &mapWd, &C.full[w], 0, B.e * p.d + nb * kStageRows, ks * sc);
                } else {
                  tma_load_3d(dst, (ks & 1) ? &mapWu : &mapWg, &C.full[w], 0, B.e * p.f + nb * kStageRows,
                              (ks >> 1) * sc);
                }
                ++issued[w];
                --left[w];
                --total;
                if (++cur_ks[w] == nks) {
                  cur_ks[w] = 0;
                  cur_i[w] += kCons;
                }
              }
            }
            if ((it & 63) == 63 && (*abort_flag || globaltimer() - t0 > kTimeoutNs)) ok = false;
          }
          u += B.n;
        }
      }
      if (!ok && atomicExch(&C.abort, 1) == 0 && p.timeouts) atomicAdd(p.timeouts, 1u);
      if (*abort_flag) {
        // drain: the latest phase of every slot must have landed before the CTA exits
        for (int w = 0; w < kCons; ++w) {
          if (issued[w] == 0) continue;
          const uint64_t t1 = globaltimer();
          while (!mbar_try_wait(&C.full[w], static_cast<uint32_t>(issued[w] - 1) & 1u) &&
                 globaltimer() - t1 < kTimeoutNs) {
          }
        }
      }
    }
  } else {
    // ===================================== consumers ====================================
    const int g = lane >> 2, q = lane & 3;
    const int rho = (g >> 1) + 4 * (g & 1);   // buffer row (and token) behind MMA row / column g
    const uint32_t slot_a = smem_u32(ring + warp * kStageBytes), x_a = smem_u32(xtile);
    int m = 0;        // stages this warp has consumed
    int blk = 0;
    bool ok = true;
    for (int phase = 0; phase < 2 && ok; ++phase) {
      const int u_end = phase ? P.b_end : P.a_end;
      const int nks = phase ? nks_b : nks_a;
      const int sc = phase ? p.sc_b : p.sc_a;
      for (int u = phase ? P.b_begin : P.a_begin; u < u_end && ok; ++blk) {
        const Block B = make_block(C, P, E, phase, u);
        // ask for this block's token tile: in phase B only once all of the expert's h rows exist
        if (phase && warp == 0 && lane == 0) {
          const unsigned int target = static_cast<unsigned int>((C.seg_a[B.e + 1] - C.seg_a[B.e]) * P.nblk_a);
          const uint64_t t0 = globaltimer();
          for (uint32_t it = 0; ld_acquire(p.ready + B.e) < target; ++it) {
            if ((it & 15) == 15 && (*abort_flag || globaltimer() - t0 > kTimeoutNs)) {
              ok = false;
              break;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;   // keep the warp uniform
        if (lane == 0) mbar_arrive(&C.x_req);
        if (!ok || !mbar_wait(&C.x_full, static_cast<uint32_t>(blk & 1), abort_flag)) {
          ok = false;
          break;
        }
        const int ng = (B.rows + 7) >> 3;
        int my_units = 0;
        for (int i = warp; i < B.n && ok; i += kCons) {
          const int nb = B.nb0 + i;
          // phase A: acc = gate, acc2 = up;  phase B: acc = h_hi part, acc2 = h_lo part.  Each
          // holds four partial sums (one per MMA position of a chunk), added up after the unit.
          float acc[3][4][4], acc2[3][4][4];
#pragma unroll
          for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int v = 0; v < 4; ++v) acc[j][r][v] = acc2[j][r][v] = 0.f;
          for (int ks = 0; ks < nks; ++ks, ++m) {
            if (!mbar_wait(&C.full[warp], static_cast<uint32_t>(m & 1), abort_flag)) {
              ok = false;
              break;
            }
            const int kc0 = phase ? ks * sc : (ks >> 1) * sc;   // first global 64-wide chunk
            const bool up = !phase && (ks & 1);
#pragma unroll 4
            for (int c = 0; c < sc; ++c) {
              uint4 a00, a01, a10, a11;   // A rows rho and rho + 8, halves k = q*8.. and 32 + q*8..
              ld_line(slot_a + (c * kStageRows + rho) * 128, rho, q, a00, a01);
              ld_line(slot_a + (c * kStageRows + rho + 8) * 128, rho, q, a10, a11);
              const int kc = kc0 + c;
              if (phase) {
                uint4 b0, b1, l0, l1;
                ld_line(x_a + (kc * kTokB + rho) * 128, rho, q, b0, b1);
                ld_line(x_a + ((kc + p.f / 64) * kTokB + rho) * 128, rho, q, l0, l1);
                mma_chunk4(acc[0], a00, a01, a10, a11, b0, b1);
                mma_chunk4(acc2[0], a00, a01, a10, a11, l0, l1);
              } else {
#pragma unroll
                for (int j = 0; j < 3; ++j) {
                  if (j < ng) {
                    uint4 b0, b1;
                    ld_line(x_a + (kc * kTokA + j * 8 + rho) * 128, rho, q, b0, b1);
                    if (up)
                      mma_chunk4(acc2[j], a00, a01, a10, a11, b0, b1);
                    else
                      mma_chunk4(acc[j], a00, a01, a10, a11, b0, b1);
                  }
                }
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&C.empty[warp]);
          }
          if (!ok) break;
          // fold the four partial sums
          float accs[3][4], accs2[3][4];
#pragma unroll
          for (int j = 0; j < 3; ++j)
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              accs[j][v] = (acc[j][0][v] + acc[j][1][v]) + (acc[j][2][v] + acc[j][3][v]);
              accs2[j][v] = (acc2[j][0][v] + acc2[j][1][v]) + (acc2[j][2][v] + acc2[j][3][v]);
            }
          // epilogue: lane (g, q) holds MMA rows g (c0, c1) and g + 8 (c2, c3), i.e. features
          // nb*16 + rho and + 8, and MMA columns 2q (c0, c2) and 2q + 1 (c1, c3) of each token
          // group, i.e. tokens rho(2q) = q and rho(2q + 1) = q + 4
          const int n0 = nb * kStageRows + rho;
          if (phase) {
            float* y = p.y;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              const int t = q + ((v & 1) ? 4 : 0);
              const int n = n0 + ((v & 2) ? 8 : 0);
              if (t < B.rows) y[static_cast<size_t>(B.row0 + t) * p.d + n] = accs[0][v] + accs2[0][v];
            }
          } else {
            const size_t ld = static_cast<size_t>(2) * p.f;
#pragma unroll
            for (int j = 0; j < 3; ++j) {
              if (j < ng) {
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                  const int t = j * 8 + q + ((v & 1) ? 4 : 0);
                  const int n = n0 + ((v & 2) ? 8 : 0);
                  if (t < B.rows) {
                    const float gt = accs[j][v], ut = accs2[j][v];
                    const float hv = gt / (1.f + expf(-gt)) * ut;
                    const uint16_t hi = f32_to_bf16_bits(hv);
                    p.h[(B.row0 + t) * ld + n] = hi;
                    p.h[(B.row0 + t) * ld + p.f + n] = f32_to_bf16_bits(hv - bf16_to_f32(hi));
                  }
                }
              }
            }
          }
          ++my_units;
        }
        if (!phase && my_units) {
          // this warp's phase-A units of the block are stored: publish them with one fence
          __syncwarp();
          if (lane == 0) red_release_add(p.ready + B.e, static_cast<unsigned int>(my_units));
        }
        u += B.n;
      }
    }
    if (!ok && lane == 0 && atomicExch(&C.abort, 1) == 0 && p.timeouts) atomicAdd(p.timeouts, 1u);
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // the token tile of the last block may still be landing
    const uint64_t t1 = globaltimer();
    while (!mbar_try_wait(&C.x_full, 0) && !mbar_try_wait(&C.x_full, 1) && globaltimer() - t1 < kTimeoutNs) {
    }
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
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
    else
      cudaGetLastError();
  }
  return fn;
}

// A bf16 matrix [rows, cols] viewed as [cols/64 chunks][rows][64], boxes of box_rows rows x
// box_chunks chunks, landing as [chunk][row][128 B] with 128-byte swizzle.
bool make_chunk_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
                    uint32_t box_chunks) {
  EncodeTiledFn enc = encoder();
  if (!enc) return false;
  const cuuint64_t dims[3] = {64, rows, cols / 64};
  const cuuint64_t strides[2] = {cols * 2, 128};
  const cuuint32_t box[3] = {64, box_rows, box_chunks};
  const cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t grouped_swiglu_decode_workspace(int E) { return static_cast<size_t>(E) * sizeof(unsigned int) + 256; }

bool grouped_swiglu_decode_supported(int d, int f) {
  // a weight stage is 1024 k (K / 64 a multiple of 16) or all of a shorter K; token tiles fit
  const bool stage_d = (d / 64) % kMaxStageChunks == 0 || d / 64 < kMaxStageChunks;
  const bool stage_f = (f / 64) % kMaxStageChunks == 0 || f / 64 < kMaxStageChunks;
  return d % 256 == 0 && f % 256 == 0 && stage_d && stage_f && kTokA * d * 2 <= kXTileBytes &&
         kTokB * 2 * f * 2 <= kXTileBytes && 2 * f / 64 <= 256 && kSmemBytes <= static_cast<size_t>(max_smem_optin());
}

// bf16 grouped SwiGLU for few rows per expert.  h: bf16 [M, 2f] (h_hi | h_lo); y_perm: f32
// [M, d]; ws: at least grouped_swiglu_decode_workspace(E) bytes (its counters are cleared here).
zmoe_status grouped_swiglu_decode(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                                  const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                                  float* y_perm, void* ws, cudaStream_t s) {
  if (!grouped_swiglu_decode_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (decode): needs d % 256 == 0, f % 256 == 0, d <= 2048, "
                                      "f <= 3072, E <= 64");
  // phase-A token tiles load in boxes of xa_box chunks; xa_box divides d / 64 (a multiple of 4).
  // A weight stage covers sc chunks of k: 16 (1024 k) when K / 64 is a multiple of 16, else all of K.
  const int nch = d / 64;
  const int sc_a = (nch % kMaxStageChunks == 0) ? kMaxStageChunks : nch;
  const int sc_b = ((f / 64) % kMaxStageChunks == 0) ? kMaxStageChunks : f / 64;
  int xa_box = 4;
  for (int b : {16, 12, 8}) {
    if (nch % b == 0) {
      xa_box = b;
      break;
    }
  }
  CUtensorMap mg, mu, md, mx, mh;
  if (!make_chunk_map(&mg, w_gate, static_cast<uint64_t>(E) * f, d, kStageRows, static_cast<uint32_t>(sc_a)) ||
      !make_chunk_map(&mu, w_up, static_cast<uint64_t>(E) * f, d, kStageRows, static_cast<uint32_t>(sc_a)) ||
      !make_chunk_map(&md, w_down, static_cast<uint64_t>(E) * d, f, kStageRows, static_cast<uint32_t>(sc_b)) ||
      !make_chunk_map(&mx, x_perm, M_total, d, kTokA, static_cast<uint32_t>(xa_box)) ||
      !make_chunk_map(&mh, h, M_total, 2 * static_cast<uint64_t>(f), kTokB, 2 * f / 64))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (decode): cuTensorMapEncodeTiled failed");
  unsigned int* ready = static_cast<unsigned int*>(ws);
  if (cudaMemsetAsync(ready, 0, static_cast<size_t>(E) * sizeof(unsigned int), s) != cudaSuccess)
    return check_launch("grouped_swiglu (decode): clearing the ready counters");
  if (cudaFuncSetAttribute(decode_ffn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kSmemBytes)) != cudaSuccess)
    return check_launch("grouped_swiglu (decode): shared memory attribute");
  DecodeArgs args{offsets, h, y_perm, ready, device_timeout_counter(), E, d, f, xa_box, sc_a, sc_b};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms()));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: the phase-B waits need it
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_ffn_kernel, mg, mu, md, mx, mh, args);
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string("grouped_swiglu (decode): ") + cudaGetErrorString(e));
  return check_launch("grouped_swiglu (decode)");
}

}  // namespace zmoe
