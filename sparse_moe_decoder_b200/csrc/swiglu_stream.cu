// Grouped SwiGLU for decode-size batches: weight streaming (HBM-bound).
//
// Per expert e (rows offsets[e]..offsets[e+1] of the permuted activations):
//   h = silu(x W_gate[e]^T) * (x W_up[e]^T)       kept as a bf16 pair h ~= h_hi + h_lo
//   y = h W_down[e]^T = h_hi W_down^T + h_lo W_down^T     (fp32)
// ("GLU Variants Improve Transformer", ZONOS2 Technical Report "Builds on"; SiLU per the
// telknet.cc article on ZONOS2, section 2.1.)
//
// With a handful of rows per expert the contraction has ~8 FLOP per weight byte: the time is
// the time to stream every touched expert's weights from HBM once.  Design:
//   * One persistent CTA per SM, 16 warps.  Work units are (expert, token chunk, 16 weight
//     rows); each CTA takes a contiguous, equal share of the unit list (computed on the device
//     from `offsets`, so no host round trip), which balances bytes per SM to within one unit.
//   * A WARP owns a whole unit: it streams the unit's 16 weight rows over the full K with
//     16-byte loads (L1::no_allocate, L2 evict-first) kept kDepth 64-wide chunks deep in
//     registers, and finishes the unit alone -- no cross-warp reduction, no barrier per unit.
//     The load cursor runs ahead across unit (and token-chunk) boundaries.
//   * Swap-AB on the tensor cores: weight rows are the MMA's M = 16, tokens are N = 8
//     (mma.sync m16n8k16, bf16 in, fp32 accumulate).  The physical k order inside a chunk is
//     permuted identically for A and B so that each lane's 16-byte load lands directly in its
//     A-fragment registers.  Only the token groups that hold rows are multiplied.
//   * The CTA stages the current (expert, token chunk) rows in shared memory (64-byte row pad:
//     conflict-free 16-byte fragment reads); it re-stages, between two CTA barriers, only when
//     its unit range crosses into the next chunk (once or twice per CTA).
//   * Gate/up units pair 8 gate rows (MMA rows 0..7) with the 8 matching up rows (rows 8..15),
//     so each lane's accumulator holds gate and up of the same (feature, token): SiLU * up is
//     applied in registers and h is stored as h_hi = bf16(h), h_lo = bf16(h - h_hi).  Down
//     units are 16 rows of W_down; each A fragment is multiplied by the h_hi and h_lo rows.
#include "common.cuh"

namespace zmoe {
namespace {

constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
constexpr int kDepth = 4;   // 64-wide K chunks per warp: one being consumed, kDepth-1 in flight
constexpr int kMaxE = 64;

enum { kGateUp = 0, kDown = 1 };

struct StreamArgs {
  const uint16_t* w0;       // gate/up: W_gate [E, R, K];  down: W_down [E, R, K]
  const uint16_t* w1;       // gate/up: W_up   [E, R, K];  down: unused
  const uint16_t* x;        // gate/up: x_perm [M, K];     down: h pair [M, 2K] (h_hi | h_lo)
  const int32_t* offsets;   // [E + 1], device
  void* out;                // gate/up: h pair bf16 [M, 2R]; down: y_perm f32 [M, R]
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

// The four MMAs of one chunk against one group of 8 token rows (b0: k = q*8.., b1: k = 32+q*8..).
__device__ __forceinline__ void mma_chunk(float (&c)[4], const Frag& f, const uint4& b0, const uint4& b1) {
  mma16816(c, f.lo0.x, f.hi0.x, f.lo0.y, f.hi0.y, b0.x, b0.y);
  mma16816(c, f.lo0.z, f.hi0.z, f.lo0.w, f.hi0.w, b0.z, b0.w);
  mma16816(c, f.lo1.x, f.hi1.x, f.lo1.y, f.hi1.y, b1.x, b1.y);
  mma16816(c, f.lo1.z, f.hi1.z, f.lo1.w, f.hi1.w, b1.z, b1.w);
}

// Unit u -> segment (expert, token chunk) index u / nblk and row block u % nblk.
__device__ __forceinline__ void seg_of(int s, const int* seg_start, const int* off, int E, int tokc, int& e,
                                       int& row0, int& rows) {
  e = 0;
  while (e + 1 < E && seg_start[e + 1] <= s) ++e;
  row0 = off[e] + (s - seg_start[e]) * tokc;
  const int left = off[e + 1] - row0;
  rows = left < tokc ? left : tokc;
}

// This lane's A row pointers (row g and row g + 8 of the unit, at k = q*8).
template <int MODE>
__device__ __forceinline__ void unit_rows(const StreamArgs& a, int e, int nb, int lane, const uint16_t*& lo,
                                          const uint16_t*& hi) {
  constexpr int FEAT = (MODE == kGateUp) ? 8 : 16;
  const int g = lane >> 2, q = lane & 3;
  const size_t row = static_cast<size_t>(e) * a.R + static_cast<size_t>(nb) * FEAT + g;
  lo = a.w0 + row * a.K + q * 8;
  hi = (MODE == kGateUp) ? a.w1 + row * a.K + q * 8 : lo + static_cast<size_t>(8) * a.K;
}

template <int MODE, int NG>
__global__ void __launch_bounds__(kThreads, 1) stream_ffn_kernel(StreamArgs a) {
  constexpr int FEAT = (MODE == kGateUp) ? 8 : 16;
  constexpr bool SPLIT = (MODE == kDown);   // the down contraction multiplies h_hi and h_lo
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __shared__ int seg_start[kMaxE + 1];
  __shared__ int off[kMaxE + 1];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, q = lane & 3;
  const int K = a.K;
  const int xld = SPLIT ? 2 * K : K;              // staged row length
  const int srow = xld + 32;                      // shared row stride (elements): conflict-free
  const int nkc = K / 64;                         // chunks per unit (a multiple of kDepth)
  const int nblk = a.R / FEAT;
  const int tokc = a.tokc;
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem_raw);   // [tokc][srow]

  if (tid <= a.E) off[tid] = a.offsets[tid];
  __syncthreads();
  if (tid == 0) {
    int acc = 0;
    for (int e = 0; e < a.E; ++e) {
      seg_start[e] = acc;
      acc += (off[e + 1] - off[e] + tokc - 1) / tokc;
    }
    seg_start[a.E] = acc;
  }
  __syncthreads();

  // unit indices fit in int: (rows / 8 + E) segments x at most d / 8 row blocks
  const int U = seg_start[a.E] * nblk;
  const int u_begin = static_cast<int>(static_cast<long long>(U) * blockIdx.x / gridDim.x);
  const int u_end = static_cast<int>(static_cast<long long>(U) * (blockIdx.x + 1) / gridDim.x);
  if (u_begin >= u_end) return;
  const int s_first = u_begin / nblk;
  const int s_last = (u_end - 1) / nblk;

  // This warp's units: in every segment s, lo(s) + warp, lo(s) + warp + 16, ... below hi(s).
  auto first_in = [&](int s) -> int {
    const int lo = max(s * nblk, u_begin);
    const int hi = min((s + 1) * nblk, u_end);
    return lo + warp < hi ? lo + warp : -1;
  };
  auto next_unit = [&](int u) -> int {
    const int s = u / nblk;
    const int hi = min((s + 1) * nblk, u_end);
    if (u + kWarps < hi) return u + kWarps;
    for (int s2 = s + 1; s2 <= s_last; ++s2) {
      const int c = first_in(s2);
      if (c >= 0) return c;
    }
    return -1;
  };

  const uint64_t pol = evict_first_policy();

  // ---- load cursor: unit lu, chunk lc ----
  int lu = -1;
  for (int s = s_first; s <= s_last && lu < 0; ++s) lu = first_in(s);
  int lc = 0;
  const uint16_t* llo = nullptr;
  const uint16_t* lhi = nullptr;
  auto point_load_cursor = [&]() {
    if (lu < 0) return;
    int e, row0, rows;
    seg_of(lu / nblk, seg_start, off, a.E, tokc, e, row0, rows);
    unit_rows<MODE>(a, e, lu % nblk, lane, llo, lhi);
  };
  point_load_cursor();
  auto issue = [&](Frag& f) {
    if (lu >= 0) {
      const int kb = lc * 64;
      f.lo0 = ldg_weights(llo + kb, pol);
      f.lo1 = ldg_weights(llo + kb + 32, pol);
      f.hi0 = ldg_weights(lhi + kb, pol);
      f.hi1 = ldg_weights(lhi + kb + 32, pol);
      if (++lc == nkc) {
        lc = 0;
        lu = next_unit(lu);
        point_load_cursor();
      }
    }
  };
  Frag buf[kDepth];
#pragma unroll
  for (int r = 0; r < kDepth; ++r) issue(buf[r]);

  // ---- segments of this CTA ----
  for (int s = s_first; s <= s_last; ++s) {
    int e, row0, rows;
    seg_of(s, seg_start, off, a.E, tokc, e, row0, rows);
    const int ng = (rows + 7) >> 3;                 // token groups that hold rows
    __syncthreads();                                // every warp is done with the previous rows
    {
      const int vpr = xld / 8;
      const uint4* src = reinterpret_cast<const uint4*>(a.x);
      for (int i = tid; i < ng * 8 * vpr; i += kThreads) {
        const int rr = i / vpr, v = i - rr * vpr;
        uint4 val = make_uint4(0u, 0u, 0u, 0u);
        if (rr < rows) val = src[static_cast<size_t>(row0 + rr) * vpr + v];
        *reinterpret_cast<uint4*>(xs + static_cast<size_t>(rr) * srow + v * 8) = val;
      }
    }
    __syncthreads();

    for (int u = first_in(s); u >= 0 && u / nblk == s; u = next_unit(u)) {
      const int nb = u % nblk;
      float acc[NG][4];
#pragma unroll
      for (int j = 0; j < NG; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;

      for (int c0 = 0; c0 < nkc; c0 += kDepth) {
#pragma unroll
        for (int r = 0; r < kDepth; ++r) {
          const Frag& f = buf[r];
          const int kb = (c0 + r) * 64;
#pragma unroll
          for (int j = 0; j < NG; ++j) {
            if (j < ng) {
              const uint16_t* xr = xs + static_cast<size_t>(j * 8 + g) * srow + kb + q * 8;
              const uint4 b0 = *reinterpret_cast<const uint4*>(xr);
              const uint4 b1 = *reinterpret_cast<const uint4*>(xr + 32);
              mma_chunk(acc[j], f, b0, b1);
              if (SPLIT) {
                const uint4 l0 = *reinterpret_cast<const uint4*>(xr + K);
                const uint4 l1 = *reinterpret_cast<const uint4*>(xr + K + 32);
                mma_chunk(acc[j], f, l0, l1);
              }
            }
          }
          issue(buf[r]);                           // refill the slot: kDepth - 1 chunks stay in flight
        }
      }

      // epilogue of the unit, straight from this warp's accumulators
#pragma unroll
      for (int j = 0; j < NG; ++j) {
        if (j < ng) {
          const int t0 = j * 8 + 2 * q, t1 = t0 + 1;
          const int n = nb * FEAT + g;
          if (MODE == kGateUp) {
            uint16_t* h = static_cast<uint16_t*>(a.out);
            const size_t ld = static_cast<size_t>(2) * a.R;
            const float h0 = acc[j][0] / (1.f + expf(-acc[j][0])) * acc[j][2];
            const float h1 = acc[j][1] / (1.f + expf(-acc[j][1])) * acc[j][3];
            const uint16_t h0_hi = f32_to_bf16_bits(h0), h1_hi = f32_to_bf16_bits(h1);
            if (t0 < rows) {
              h[(row0 + t0) * ld + n] = h0_hi;
              h[(row0 + t0) * ld + a.R + n] = f32_to_bf16_bits(h0 - bf16_to_f32(h0_hi));
            }
            if (t1 < rows) {
              h[(row0 + t1) * ld + n] = h1_hi;
              h[(row0 + t1) * ld + a.R + n] = f32_to_bf16_bits(h1 - bf16_to_f32(h1_hi));
            }
          } else {
            float* y = static_cast<float*>(a.out);
            if (t0 < rows) {
              y[static_cast<size_t>(row0 + t0) * a.R + n] = acc[j][0];
              y[static_cast<size_t>(row0 + t0) * a.R + n + 8] = acc[j][2];
            }
            if (t1 < rows) {
              y[static_cast<size_t>(row0 + t1) * a.R + n] = acc[j][1];
              y[static_cast<size_t>(row0 + t1) * a.R + n + 8] = acc[j][3];
            }
          }
        }
      }
    }
  }
}

size_t stream_smem_bytes(int xld, int tokc) { return static_cast<size_t>(tokc) * (xld + 32) * 2; }

// Largest token chunk (multiple of 8, <= 24: three token groups keep the kernel within 128
// registers) whose staged rows fit the device's shared memory.
int pick_tokc(int xld) {
  const size_t cap = static_cast<size_t>(max_smem_optin()) - 1024;   // static smem of the kernel
  for (int tokc = 24; tokc >= 8; tokc -= 8)
    if (stream_smem_bytes(xld, tokc) <= cap) return tokc;
  return 0;
}

template <int MODE, int NG>
zmoe_status launch_stream_ng(const StreamArgs& a, cudaStream_t s) {
  auto kern = stream_ffn_kernel<MODE, NG>;
  const size_t smem = stream_smem_bytes(MODE == kDown ? 2 * a.K : a.K, a.tokc);
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
    default: return launch_stream_ng<MODE, 3>(a, s);
  }
}

}  // namespace

bool grouped_swiglu_stream_supported(int d, int f) {
  return d % (64 * kDepth) == 0 && f % (64 * kDepth) == 0 && pick_tokc(d) > 0 && pick_tokc(2 * f) > 0;
}

// bf16 grouped SwiGLU by weight streaming (any rows per expert; efficient up to one token chunk).
// h: bf16 [M, 2f] (h_hi | h_lo); y_perm: f32 [M, d].
zmoe_status grouped_swiglu_stream(const uint16_t* x_perm, const int32_t* offsets, const uint16_t* w_gate,
                                  const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                                  float* y_perm, cudaStream_t s) {
  if (!grouped_swiglu_stream_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (stream): needs d % 256 == 0, f % 256 == 0, E <= 64");
  StreamArgs gu{w_gate, w_up, x_perm, offsets, h, E, d, f, pick_tokc(d)};
  StreamArgs dn{w_down, nullptr, h, offsets, y_perm, E, f, d, pick_tokc(2 * f)};
  zmoe_status st = launch_stream<kGateUp>(gu, s);
  if (st != ZMOE_OK) return st;
  return launch_stream<kDown>(dn, s);
}

}  // namespace zmoe
