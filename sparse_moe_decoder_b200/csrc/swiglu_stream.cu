// Grouped SwiGLU for decode-size batches: weight streaming (HBM-bound).
//
// Per expert e (rows offsets[e]..offsets[e+1] of the permuted activations):
//   h = silu(x W_gate[e]^T) * (x W_up[e]^T)      (bf16, the operand of the next contraction)
//   y = h W_down[e]^T                              (fp32)
// ("GLU Variants Improve Transformer", ZONOS2 Technical Report "Builds on"; SiLU per the
// telknet.cc article on ZONOS2, section 2.1.)
//
// With a handful of rows per expert the contraction has ~8 FLOP per weight byte: the time is
// the time to stream every touched expert's weights from HBM once.  Design:
//   * One persistent CTA per SM, 16 warps.  Work units are (expert, token chunk, 16 weight
//     rows); each CTA takes a contiguous, equal share of the unit list (read on the device from
//     `offsets`, so no host round trip), which keeps every SM's byte count within one unit.
//   * A unit's K range is dealt in 64-wide chunks round-robin to the 16 warps; a warp loads its
//     weight fragments straight from global memory with 16-byte streaming loads
//     (L1::no_allocate, L2 evict-first) and keeps kDepth chunks in flight (~96 KB per SM).
//   * Swap-AB on the tensor cores: weight rows are the MMA's M = 16, tokens are N = 8
//     (mma.sync m16n8k16, bf16 in, fp32 accumulate).  The physical k order inside a chunk is
//     permuted identically for A and B so that each lane's 16-byte load lands directly in its
//     A-fragment registers; the token rows (B) sit in shared memory with a 64-byte row pad
//     that makes the 16-byte fragment reads bank-conflict free.
//   * Gate/up units pair 8 gate rows (MMA rows 0..7) with the 8 matching up rows (rows 8..15),
//     so each lane's accumulator holds gate and up of the same (feature, token): SiLU * up is
//     applied in registers in the epilogue.  Down units are 16 rows of W_down.
//   * The 16 warps' partial sums are added through shared memory (double-buffered, one CTA
//     barrier per unit).
#include "common.cuh"

namespace zmoe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kDepth = 4;   // 64-wide K chunks per warp: one being consumed, kDepth-1 in flight
constexpr int kMaxE = 64;

enum { kGateUp = 0, kDown = 1 };

struct StreamArgs {
  const uint16_t* a0;       // gate/up: W_gate [E, R, K];  down: W_down [E, R, K]
  const uint16_t* a1;       // gate/up: W_up   [E, R, K];  down: unused
  const uint16_t* x;        // gate/up: x_perm [M, K];     down: h [M, K]
  const int32_t* offsets;   // [E + 1], device
  void* out;                // gate/up: h bf16 [M, R];     down: y_perm f32 [M, R]
  int E, K, R, tokc;
};

__device__ __forceinline__ uint64_t evict_first_policy() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ uint4 ldg_weights(const uint16_t* ptr, uint64_t pol) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(ptr), "l"(pol));
  return r;
}

__device__ __forceinline__ void mma16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// The A fragments of one 64-wide chunk for one lane: rows g (lo) and g + 8 (hi), physical
// k = q*8 .. q*8+7 (v0) and 32 + q*8 .. +7 (v1) of the chunk.
struct Frag {
  uint4 lo0, lo1, hi0, hi1;
};

// Position of a unit in the (expert, chunk, row block) grid, plus its row pointers.
struct UnitPos {
  int e, chunk, nb;
  int row0, rows;               // first permuted row of the chunk, rows in it (<= tokc)
  const uint16_t* lo;           // this lane's A row g at k = q*8
  const uint16_t* hi;           // this lane's A row g + 8 at k = q*8
};

template <int MODE>
__device__ __forceinline__ UnitPos locate(long long u, const int* unit_start, const int* off, const StreamArgs& a,
                                          int nblk, int lane) {
  constexpr int FEAT = (MODE == kGateUp) ? 8 : 16;
  UnitPos p;
  int e = 0;
  while (e + 1 < a.E && unit_start[e + 1] <= u) ++e;
  const int local = static_cast<int>(u - unit_start[e]);
  p.e = e;
  p.chunk = local / nblk;
  p.nb = local - p.chunk * nblk;
  p.row0 = off[e] + p.chunk * a.tokc;
  const int left = off[e + 1] - p.row0;
  p.rows = left < a.tokc ? left : a.tokc;
  const int g = lane >> 2, q = lane & 3;
  const size_t row = static_cast<size_t>(e) * a.R + static_cast<size_t>(p.nb) * FEAT + g;
  p.lo = a.a0 + row * a.K + q * 8;
  p.hi = (MODE == kGateUp) ? a.a1 + row * a.K + q * 8 : p.lo + static_cast<size_t>(8) * a.K;
  return p;
}

template <int MODE, int NG>
__global__ void __launch_bounds__(kThreads, 1) stream_ffn_kernel(StreamArgs a) {
  constexpr int FEAT = (MODE == kGateUp) ? 8 : 16;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int unit_start[kMaxE + 1];
  __shared__ int off[kMaxE + 1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int K = a.K;
  const int srow = K + 32;                       // shared row stride (elements): conflict-free
  const int nkc = K / 64;                        // 64-wide chunks per unit
  const int per = (nkc + kWarps - 1) / kWarps;   // chunk slots per warp per unit
  const int nblk = a.R / FEAT;
  const int tokc = a.tokc;

  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw);                                     // [tokc][srow]
  float4* red = reinterpret_cast<float4*>(smem_raw + static_cast<size_t>(tokc) * srow * 2);  // [2][16][NG][32]

  if (tid <= a.E) off[tid] = a.offsets[tid];
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < a.E; ++e) {
      unit_start[e] = acc;
      const int m = off[e + 1] - off[e];
      acc += ((m + tokc - 1) / tokc) * nblk;
    }
    unit_start[a.E] = acc;
  }
  __syncthreads();

  const long long U = unit_start[a.E];
  const long long u_begin = U * blockIdx.x / gridDim.x;
  const long long u_end = U * (blockIdx.x + 1) / gridDim.x;
  const long long S = (u_end - u_begin) * per;   // chunk slots this warp walks through
  if (S == 0) return;

  const uint64_t pol = evict_first_policy();

  // load cursor (runs kDepth slots ahead of the compute cursor)
  long long lu = u_begin;
  int lj = 0;
  UnitPos lp = locate<MODE>(lu, unit_start, off, a, nblk, lane);

  auto issue = [&](Frag& f) {
    const int kc = warp + kWarps * lj;
    if (lu < u_end && kc < nkc) {
      const int kb = kc * 64;
      f.lo0 = ldg_weights(lp.lo + kb, pol);
      f.lo1 = ldg_weights(lp.lo + kb + 32, pol);
      f.hi0 = ldg_weights(lp.hi + kb, pol);
      f.hi1 = ldg_weights(lp.hi + kb + 32, pol);
    }
    if (++lj == per) {
      lj = 0;
      ++lu;
      if (lu < u_end) lp = locate<MODE>(lu, unit_start, off, a, nblk, lane);
    }
  };

  Frag buf[kDepth];
#pragma unroll
  for (int r = 0; r < kDepth; ++r) issue(buf[r]);

  // compute cursor
  long long cu = u_begin;
  int cj = 0;
  UnitPos cp;
  int tile_e = -1, tile_chunk = -1;
  int parity = 0;
  float acc[NG][4];
#pragma unroll
  for (int j = 0; j < NG; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

  for (long long s0 = 0; s0 < S; s0 += kDepth) {
#pragma unroll
    for (int r = 0; r < kDepth; ++r) {
      if (s0 + r < S) {
        if (cj == 0) {
          cp = locate<MODE>(cu, unit_start, off, a, nblk, lane);
          if (cp.e != tile_e || cp.chunk != tile_chunk) {
            // Stage this chunk's token rows (zero-padded to tokc).  Every warp has passed the
            // previous unit's barrier, so nobody still reads the old tile.
            const int vpr = K / 8;
            const uint4* src = reinterpret_cast<const uint4*>(a.x);
            for (int i = tid; i < tokc * vpr; i += kThreads) {
              const int rr = i / vpr, v = i - rr * vpr;
              uint4 val = make_uint4(0u, 0u, 0u, 0u);
              if (rr < cp.rows) val = src[static_cast<size_t>(cp.row0 + rr) * vpr + v];
              *reinterpret_cast<uint4*>(xs + static_cast<size_t>(rr) * srow + v * 8) = val;
            }
            tile_e = cp.e;
            tile_chunk = cp.chunk;
            __syncthreads();
          }
        }
        const int kc = warp + kWarps * cj;
        if (kc < nkc) {
          const Frag& f = buf[r];
          const int kb = kc * 64;
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            const uint16_t* xr = xs + static_cast<size_t>(j * 8 + g) * srow + kb + q * 8;
            const uint4 b0 = *reinterpret_cast<const uint4*>(xr);
            const uint4 b1 = *reinterpret_cast<const uint4*>(xr + 32);
            mma16816(acc[j], f.lo0.x, f.hi0.x, f.lo0.y, f.hi0.y, b0.x, b0.y);
            mma16816(acc[j], f.lo0.z, f.hi0.z, f.lo0.w, f.hi0.w, b0.z, b0.w);
            mma16816(acc[j], f.lo1.x, f.hi1.x, f.lo1.y, f.hi1.y, b1.x, b1.y);
            mma16816(acc[j], f.lo1.z, f.hi1.z, f.lo1.w, f.hi1.w, b1.z, b1.w);
          }
        }
        issue(buf[r]);
        if (++cj == per) {
          // end of unit: reduce the 16 warps' partial sums and write the outputs
          float4* rb = red + static_cast<size_t>(parity) * kWarps * NG * 32;
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            rb[(warp * NG + j) * 32 + lane] = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
            acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
          }
          __syncthreads();
          if (tid < NG * 32) {
            const int j = tid >> 5;
            float4 c = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int w = 0; w < kWarps; ++w) {
              const float4 v = rb[(w * NG + j) * 32 + lane];
              c.x += v.x;
              c.y += v.y;
              c.z += v.z;
              c.w += v.w;
            }
            const int t0 = j * 8 + 2 * q, t1 = t0 + 1;
            const int n = cp.nb * FEAT + g;
            if (MODE == kGateUp) {
              uint16_t* h = static_cast<uint16_t*>(a.out);
              if (t0 < cp.rows) h[static_cast<size_t>(cp.row0 + t0) * a.R + n] = f32_to_bf16_bits(c.x / (1.f + expf(-c.x)) * c.z);
              if (t1 < cp.rows) h[static_cast<size_t>(cp.row0 + t1) * a.R + n] = f32_to_bf16_bits(c.y / (1.f + expf(-c.y)) * c.w);
            } else {
              float* y = static_cast<float*>(a.out);
              if (t0 < cp.rows) {
                y[static_cast<size_t>(cp.row0 + t0) * a.R + n] = c.x;
                y[static_cast<size_t>(cp.row0 + t0) * a.R + n + 8] = c.z;
              }
              if (t1 < cp.rows) {
                y[static_cast<size_t>(cp.row0 + t1) * a.R + n] = c.y;
                y[static_cast<size_t>(cp.row0 + t1) * a.R + n + 8] = c.w;
              }
            }
          }
          parity ^= 1;
          cj = 0;
          ++cu;
        }
      }
    }
  }
}

size_t stream_smem_bytes(int K, int tokc) {
  const int ng = tokc / 8;
  return static_cast<size_t>(tokc) * (K + 32) * 2 + static_cast<size_t>(2) * kWarps * ng * 32 * sizeof(float4);
}

// Largest token chunk (multiple of 8, <= 32) whose tile fits the device's shared memory.
int pick_tokc(int K) {
  const size_t cap = static_cast<size_t>(max_smem_optin()) - 1024;   // static smem of the kernel
  for (int tokc = 32; tokc >= 8; tokc -= 8)
    if (stream_smem_bytes(K, tokc) <= cap) return tokc;
  return 0;
}

template <int MODE, int NG>
zmoe_status launch_stream_ng(const StreamArgs& a, cudaStream_t s) {
  auto kern = stream_ffn_kernel<MODE, NG>;
  const size_t smem = stream_smem_bytes(a.K, a.tokc);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) != cudaSuccess)
    return check_launch("grouped_swiglu (stream): shared memory attribute");
  kern<<<num_sms(), kThreads, smem, s>>>(a);
  return check_launch("grouped_swiglu (stream)");
}

template <int MODE>
zmoe_status launch_stream(const StreamArgs& a, cudaStream_t s) {
  switch (a.tokc / 8) {
    case 1: return launch_stream_ng<MODE, 1>(a, s);
    case 2: return launch_stream_ng<MODE, 2>(a, s);
    case 3: return launch_stream_ng<MODE, 3>(a, s);
    default: return launch_stream_ng<MODE, 4>(a, s);
  }
}

}  // namespace

// bf16 grouped SwiGLU by weight streaming (any rows per expert; efficient for <= 32).
zmoe_status grouped_swiglu_stream(const uint16_t* x_perm, const int32_t* offsets, const uint16_t* w_gate,
                                  const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                                  float* y_perm, cudaStream_t s) {
  if (d % 64 != 0 || f % 64 != 0 || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (stream): needs d % 64 == 0, f % 64 == 0, E <= 64");
  StreamArgs gu{w_gate, w_up, x_perm, offsets, h, E, d, f, pick_tokc(d)};
  StreamArgs dn{w_down, nullptr, h, offsets, y_perm, E, f, d, pick_tokc(f)};
  if (gu.tokc == 0 || dn.tokc == 0) return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (stream): d or f too large");
  zmoe_status st = launch_stream<kGateUp>(gu, s);
  if (st != ZMOE_OK) return st;
  return launch_stream<kDown>(dn, s);
}

}  // namespace zmoe
