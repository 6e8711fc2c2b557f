// Grouped SwiGLU for decode-size batches on the tensor cores: swap-AB, stream-K, one launch.
//
// Per expert e over its rows of the permuted activations ("GLU Variants Improve Transformer",
// ZONOS2 Technical Report "Builds on"; SiLU per the telknet.cc article on ZONOS2, section 2.1):
//   phase A (gate/up): h = silu(x W_gate[e]^T) * (x W_up[e]^T), stored as the bf16 pair
//                      h_hi = bf16(h), h_lo = bf16(h - h_hi)
//   phase B (down):    y_perm = h_hi W_down[e]^T + h_lo W_down[e]^T          (fp32)
//
// With a few rows per expert the work is streaming the touched experts' weights from HBM once.
// Design:
//   * Swap-AB on tcgen05: 128 weight rows are the MMA's M, a block of up to 16 token rows is its N
//     (kind::f16, bf16 in, fp32 accumulate in TMEM).  A unit is (expert, 128-row weight block, token
//     block); its k-range is cut into 256-wide stages (a 64 KB weight box + an 8/16 KB token box).
//   * Stream-K: every CTA (one per SM, cooperative launch: all resident) takes an equal,
//     contiguous range of the stage list of each phase, so bytes per SM balance to within one
//     stage whatever the expert loads are (down to a single expert at batch 1).  A unit wholly
//     inside a CTA's range is finished in TMEM; a unit cut by a range edge leaves fp32 partial
//     sums in a per-CTA slot and the last CTA to arrive adds the partials in CTA order
//     (deterministic) and finishes it.  Each CTA runs its (at most two) cut units first, so the
//     cross-CTA hand-offs overlap the whole units that follow.
//   * Roles: warp 0 loads weight boxes and warp 6 token boxes (x, or the h pair) with TMA into a
//     2-stage ring (160 KB; a 64 KB box is the size at which one SM's TMA reaches full HBM rate),
//     each completing on its own mbarrier, so weight loads never wait for h; warp 1 allocates TMEM
//     and issues the MMAs from one thread (tcgen05.commit frees a stage when its MMAs are done);
//     warps 2..5 read the accumulators with tcgen05.ld and run the epilogues.
//   * Phase-A units of expert e release-increment ready[e]; the token producer acquires ready[e]
//     before loading h rows of expert e (cross-proxy fence before the TMA).
//   * Every wait is bounded (time limit): on expiry the CTA counts a device timeout, aborts,
//     drains its own copies and MMAs, frees its TMEM and returns.
#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int BM = 128;                       // weight rows per unit (MMA M)
constexpr int NT = 16;                        // token rows per block (MMA N)
constexpr int KS = 256;                       // k per stage
constexpr int CH = KS / 64;                   // 64-wide chunks per stage
constexpr int STAGES = 2;
constexpr int W_BYTES = BM * KS * 2;          // 64 KB
constexpr int X_BYTES = NT * KS * 2;          // 8 KB  x slice
constexpr int HP_BYTES = NT * KS * 2 * 2;     // 16 KB h_hi + h_lo slice
constexpr int STAGE_BYTES = W_BYTES + HP_BYTES;
constexpr int kThreads = 224;                 // 7 warps
constexpr int kWarpTok = 6;
constexpr uint32_t TMEM_COLS = 64;            // 2 accumulator buffers x (gate 16 | up 16)
constexpr int kMaxE = 64;
constexpr int kMaxCtas = 256;
constexpr unsigned long long kTimeoutNs = 2000000000ull;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, NT);

struct DecArgs {
  const int32_t* offsets;   // [E + 1]
  uint16_t* h;              // [M, 2f] h_hi | h_lo
  float* y;                 // [M, d]
  unsigned int* ready;      // [E]    finished phase-A units per expert
  unsigned int* cnt_a;      // [ua]   arrivals per cut phase-A unit
  unsigned int* cnt_b;      // [ub]
  float* part_a;            // [C][2 slots][2 mats][NT][BM] partial sums of cut phase-A units
  float* part_b;            // [C][2 slots][NT][BM]
  unsigned int* timeouts;
  unsigned int* errors;
  int E, d, f, M_total;
  int ua_cap, ub_cap;       // units the counter arrays hold
};

struct __align__(8) Ctrl {
  uint64_t full_w[STAGES];
  uint64_t full_t[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int bad;
  int last_flag;
  int off[kMaxE + 1];
  int ustart[2][kMaxE + 1];  // first unit of each expert, per phase
  int rlo[2][kMaxCtas + 1];  // first stage of each CTA's range, per phase
};

constexpr size_t kSmemBytes = 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES + sizeof(Ctrl);

// ------------------------------------------------------------------------------------------
// work geometry (every role walks the same sequence)
// ------------------------------------------------------------------------------------------
struct Unit {
  int e, rb, row0, rows;    // expert, weight block, first permuted row, rows in the token block
};

__device__ __forceinline__ Unit unit_of(const Ctrl& C, int ph, int E, int u) {
  const int* us = C.ustart[ph];
  int e = 0;
  while (e + 1 < E && us[e + 1] <= u) ++e;
  const int ntb = (C.off[e + 1] - C.off[e] + NT - 1) / NT;
  const int local = u - us[e];
  Unit U;
  U.e = e;
  U.rb = local / ntb;
  const int tb = local - U.rb * ntb;
  U.row0 = C.off[e] + tb * NT;
  const int left = C.off[e + 1] - U.row0;
  U.rows = left < NT ? left : NT;
  return U;
}

// A CTA's stage range [sb, se) as segments (one unit each): the cut first and last units, then the
// whole units in order.
struct Plan {
  int sb, se, S, uf, ul, pf, pl, w0, n;
};

struct Seg {
  int u, j0, j1;
};

__device__ __forceinline__ Plan make_plan(int sb, int se, int S) {
  Plan P{sb, se, S, 0, 0, 0, 0, 0, 0};
  if (se <= sb) return P;
  P.uf = sb / S;
  P.ul = (se - 1) / S;
  if (P.uf == P.ul) {
    P.n = 1;
    return P;
  }
  P.pf = (sb % S) != 0;
  P.pl = (se % S) != 0;
  P.w0 = P.pf ? P.uf + 1 : P.uf;
  const int w1 = P.pl ? P.ul - 1 : P.ul;
  P.n = P.pf + P.pl + (w1 - P.w0 + 1);
  return P;
}

__device__ __forceinline__ Seg seg_at(const Plan& P, int i) {
  if (P.uf == P.ul) return Seg{P.uf, P.sb - P.uf * P.S, P.se - P.uf * P.S};
  if (P.pf) {
    if (i == 0) return Seg{P.uf, P.sb - P.uf * P.S, P.S};
    --i;
  }
  if (P.pl) {
    if (i == 0) return Seg{P.ul, 0, P.se - P.ul * P.S};
    --i;
  }
  return Seg{P.w0 + i, 0, P.S};
}

// The CTA whose range holds stage s (the largest c with rlo[c] <= s; its range is not empty).
__device__ __forceinline__ int cta_of(const int* rlo, int nC, int s) {
  int lo = 0, hi = nC - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (rlo[mid] <= s) lo = mid;
    else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ void set_abort(Ctrl& C, unsigned int* counter) {
  if (atomicExch(&C.abort, 1) == 0 && counter) atomicAdd(counter, 1u);
}

// Named barrier 1 joins the four epilogue warps.
__device__ __forceinline__ void epi_bar() { bar_sync(1, 128); }

// Waits until the latest armed phase of each slot of `bars` has completed (bounded).
__device__ __forceinline__ void drain_ring(uint64_t* bars, int armed) {
  for (int sl = 0; sl < STAGES; ++sl) {
    const int last = armed - 1 - (((armed - 1 - sl) % STAGES) + STAGES) % STAGES;
    if (last < 0) continue;
    const uint64_t t1 = globaltimer();
    while (!mbar_try_wait(&bars[sl], static_cast<uint32_t>((last / STAGES) & 1)) && globaltimer() - t1 < kTimeoutNs) {
    }
  }
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    dec_tc_kernel(const __grid_constant__ CUtensorMap mapWg, const __grid_constant__ CUtensorMap mapWu,
                  const __grid_constant__ CUtensorMap mapWd, const __grid_constant__ CUtensorMap mapX,
                  const __grid_constant__ CUtensorMap mapH, DecArgs p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctrl& C = *reinterpret_cast<Ctrl*>(base + STAGES * STAGE_BYTES);
  volatile int* abort_flag = &C.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int nC = gridDim.x, cta = blockIdx.x;
  const int S[2] = {2 * (p.d / KS), p.f / KS};   // stages per unit; phase A alternates gate / up along k

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&C.full_w[s], 1);
      mbar_init(&C.full_t[s], 1);
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
  for (int i = threadIdx.x; i <= E; i += blockDim.x) C.off[i] = p.offsets[i];
  if (warp == 1) tmem_alloc(&C.tmem_base, TMEM_COLS);
  __syncthreads();
  if (threadIdx.x == 0) {
    // offsets must be a monotone split of [0, M_total); anything else is refused before any access
    int bad = C.off[0] != 0 || C.off[E] > p.M_total;
    int a = 0, b = 0;
    for (int e = 0; e < E; ++e) {
      bad |= C.off[e + 1] < C.off[e];
      const int ntb = bad ? 0 : (C.off[e + 1] - C.off[e] + NT - 1) / NT;
      C.ustart[0][e] = a;
      C.ustart[1][e] = b;
      a += ntb * (p.f / BM);
      b += ntb * (p.d / BM);
    }
    C.ustart[0][E] = a;
    C.ustart[1][E] = b;
    bad |= a > p.ua_cap || b > p.ub_cap;
    C.bad = bad;
    if (bad && cta == 0) record_device_error(p.errors);
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= nC; i += blockDim.x) {
    C.rlo[0][i] = static_cast<int>(static_cast<long long>(C.ustart[0][E]) * S[0] * i / nC);
    C.rlo[1][i] = static_cast<int>(static_cast<long long>(C.ustart[1][E]) * S[1] * i / nC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = C.tmem_base;
  if (C.bad) {
    if (warp == 1) tmem_dealloc(tmem, TMEM_COLS);
    return;
  }

  if (warp == 0 || warp == kWarpTok) {
    // ============================ producers: weights (warp 0), tokens (warp 6) ============================
    if (lane == 0) {
      const bool wt = warp == 0;
      uint64_t* full = wt ? C.full_w : C.full_t;
      int q = 0;            // stages armed on `full`
      bool ok = true;
      int ready_e = -1;     // last expert whose phase-A units were all seen complete
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Plan P = make_plan(C.rlo[ph][cta], C.rlo[ph][cta + 1], S[ph]);
        for (int i = 0; i < P.n && ok; ++i) {
          const Seg g = seg_at(P, i);
          const Unit U = unit_of(C, ph, E, g.u);
          for (int j = g.j0; j < g.j1; ++j) {
            const int slot = q % STAGES;
            if (!mbar_wait(&C.empty[slot], static_cast<uint32_t>((q / STAGES) & 1) ^ 1u, abort_flag, kTimeoutNs)) {
              ok = false;
              break;
            }
            unsigned char* dst = base + slot * STAGE_BYTES;
            if (wt) {
              mbar_expect_tx(&full[slot], W_BYTES);
              if (ph == 0)
                tma_load_3d(dst, (j & 1) ? &mapWu : &mapWg, &full[slot], 0, U.e * p.f + U.rb * BM, (j >> 1) * CH);
              else
                tma_load_3d(dst, &mapWd, &full[slot], 0, U.e * p.d + U.rb * BM, j * CH);
            } else if (ph == 0) {
              mbar_expect_tx(&full[slot], X_BYTES);
              tma_load_3d(dst + W_BYTES, &mapX, &full[slot], 0, U.row0, (j >> 1) * CH);
            } else {
              if (U.e != ready_e) {
                // every phase-A unit of expert e must have stored its h rows
                const unsigned int target = static_cast<unsigned int>(C.ustart[0][U.e + 1] - C.ustart[0][U.e]);
                const uint64_t t0 = globaltimer();
                for (uint32_t it = 0; ld_acquire(p.ready + U.e) < target; ++it) {
                  if ((it & 15) == 15 && (*abort_flag || globaltimer() - t0 > kTimeoutNs)) {
                    ok = false;
                    break;
                  }
                }
                if (!ok) break;
                ready_e = U.e;
                asm volatile("fence.proxy.async.global;" ::: "memory");
              }
              mbar_expect_tx(&full[slot], HP_BYTES);
              tma_load_4d(dst + W_BYTES, &mapH, &full[slot], 0, U.row0, 0, j * CH);
            }
            ++q;
          }
        }
      }
      if (!ok) set_abort(C, p.timeouts);
      if (*abort_flag) drain_ring(full, q);   // no copy may land after the CTA has gone
    }
  } else if (warp == 1) {
    // ===================================== MMA issuer =====================================
    if (lane == 0) {
      int q = 0;     // stages consumed
      int seg = 0;   // segments (accumulator uses)
      bool ok = true;
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Plan P = make_plan(C.rlo[ph][cta], C.rlo[ph][cta + 1], S[ph]);
        for (int i = 0; i < P.n && ok; ++i) {
          const Seg g = seg_at(P, i);
          const int b = seg & 1;
          if (!mbar_wait(&C.tempty[b], static_cast<uint32_t>((seg >> 1) & 1) ^ 1u, abort_flag, kTimeoutNs)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int j = g.j0; j < g.j1; ++j, ++q) {
            const int slot = q % STAGES;
            const uint32_t par = static_cast<uint32_t>((q / STAGES) & 1);
            if (!mbar_wait(&C.full_w[slot], par, abort_flag, kTimeoutNs) ||
                !mbar_wait(&C.full_t[slot], par, abort_flag, kTimeoutNs)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(base + slot * STAGE_BYTES);
            const uint32_t sb = sa + W_BYTES;
            if (ph == 0) {
              // gate and up stages alternate: the first stage of each matrix in the segment is one of
              // the first two, and its first MMA overwrites that accumulator
              const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * 32 + (j & 1) * 16);
              const bool fresh = j - g.j0 < 2;
#pragma unroll
              for (int c = 0; c < CH; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                  umma_bf16(d_tmem, sw128_desc(sa + c * (BM * 128) + kk * 32), sw128_desc(sb + c * (NT * 128) + kk * 32),
                            kIdesc, (fresh && c == 0 && kk == 0) ? 0u : 1u);
            } else {
              // h_hi and h_lo slices of chunk c sit at 2c and 2c + 1 (2 KB each)
              const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * 32);
              const bool fresh = j == g.j0;
#pragma unroll
              for (int c = 0; c < CH; ++c)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t ad = sw128_desc(sa + c * (BM * 128) + kk * 32);
                  umma_bf16(d_tmem, ad, sw128_desc(sb + (2 * c) * (NT * 128) + kk * 32), kIdesc,
                            (fresh && c == 0 && kk == 0) ? 0u : 1u);
                  umma_bf16(d_tmem, ad, sw128_desc(sb + (2 * c + 1) * (NT * 128) + kk * 32), kIdesc, 1u);
                }
            }
            umma_commit(&C.empty[slot]);
          }
          if (!ok) break;
          umma_commit(&C.tfull[b]);
          ++seg;
        }
      }
      if (!ok) set_abort(C, p.timeouts);
      // every MMA this thread issued completes before the drain barrier flips
      umma_commit(&C.drain);
      const uint64_t t1 = globaltimer();
      while (!mbar_try_wait(&C.drain, 0) && globaltimer() - t1 < kTimeoutNs) {
      }
    }
  } else {
    // ===================================== epilogue (warps 2..5) =====================================
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;                 // accumulator row = TMEM lane
    const int et = threadIdx.x - 64;                     // 0..127 in the epilogue group
    int seg = 0;
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Plan P = make_plan(C.rlo[ph][cta], C.rlo[ph][cta + 1], S[ph]);
      const int* rlo = C.rlo[ph];
      for (int i = 0; i < P.n; ++i) {
        const Seg sg = seg_at(P, i);
        const int b = seg & 1;
        // all four warps take the same branch (a warp alone at a named barrier would never leave it)
        ok = bar_and(1, 128, mbar_wait(&C.tfull[b], static_cast<uint32_t>((seg >> 1) & 1), abort_flag, kTimeoutNs));
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(b * 32);
        float g[NT], v[NT];
        {
          uint32_t r0[16], r1[16];
          tmem_ld16(taddr, r0);
          if (ph == 0) tmem_ld16(taddr + 16, r1);
          tmem_wait_ld();
          // a segment without gate (up) stages left that accumulator untouched: it contributes 0
          const bool has_g = ph == 1 || sg.j0 < sg.j1 - 1 || (sg.j0 & 1) == 0;
          const bool has_u = ph == 0 && (sg.j0 < sg.j1 - 1 || (sg.j0 & 1) == 1);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            g[t] = has_g ? __uint_as_float(r0[t]) : 0.f;
            v[t] = has_u ? __uint_as_float(r1[t]) : 0.f;
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&C.tempty[b]);
        ++seg;

        const Unit U = unit_of(C, ph, E, sg.u);
        if (!(sg.j0 == 0 && sg.j1 == P.S)) {
          // leave this CTA's partial sums, then let the last contributor finish the unit
          const size_t part_elems = static_cast<size_t>(ph == 0 ? 2 : 1) * NT * BM;
          float* const part = ph == 0 ? p.part_a : p.part_b;
          {
            float* pp = part + (static_cast<size_t>(cta) * 2 + (rlo[cta] / P.S == sg.u ? 0 : 1)) * part_elems;
#pragma unroll
            for (int t = 0; t < NT; ++t)
              if (t < U.rows) {
                pp[t * BM + row] = g[t];
                if (ph == 0) pp[NT * BM + t * BM + row] = v[t];
              }
          }
          const int c_first = cta_of(rlo, nC, sg.u * P.S);
          const int c_last = cta_of(rlo, nC, (sg.u + 1) * P.S - 1);
          int ncontrib = 0;
          for (int c2 = c_first; c2 <= c_last; ++c2) ncontrib += rlo[c2 + 1] > rlo[c2];
          epi_bar();
          if (et == 0) {
            unsigned int* cnt = (ph ? p.cnt_b : p.cnt_a) + sg.u;
            C.last_flag = (atom_acq_rel_add(cnt, 1u) == static_cast<unsigned int>(ncontrib - 1)) ? 1 : 0;
          }
          epi_bar();
          if (!C.last_flag) continue;
          // sum the contributions in CTA order, two contributors' loads in flight at a time
#pragma unroll
          for (int t = 0; t < NT; ++t) g[t] = v[t] = 0.f;
          for (int c2 = c_first; c2 <= c_last; c2 += 2) {
            float ga[2][NT], va[2][NT];
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int c3 = c2 + k;
              const bool live = c3 <= c_last && rlo[c3 + 1] > rlo[c3];
              const float* pp =
                  part + (static_cast<size_t>(live ? c3 : cta) * 2 + (live && rlo[c3] / P.S == sg.u ? 0 : 1)) * part_elems;
#pragma unroll
              for (int t = 0; t < NT; ++t) {
                const bool in = live && t < U.rows;
                ga[k][t] = in ? __ldcg(pp + t * BM + row) : 0.f;
                va[k][t] = (in && ph == 0) ? __ldcg(pp + NT * BM + t * BM + row) : 0.f;
              }
            }
#pragma unroll
            for (int k = 0; k < 2; ++k)
#pragma unroll
              for (int t = 0; t < NT; ++t) {
                g[t] += ga[k][t];
                v[t] += va[k][t];
              }
          }
        }
        // the unit's final epilogue
        const int n = U.rb * BM + row;
        if (ph == 0) {
          const size_t ld = static_cast<size_t>(2) * p.f;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            if (t < U.rows) {
              const float hv = g[t] / (1.f + expf(-g[t])) * v[t];
              const uint16_t hi = f32_to_bf16_bits(hv);
              uint16_t* hr = p.h + static_cast<size_t>(U.row0 + t) * ld;
              hr[n] = hi;
              hr[p.f + n] = f32_to_bf16_bits(hv - bf16_to_f32(hi));
            }
          }
          epi_bar();
          if (et == 0) red_release_add(p.ready + U.e, 1u);
        } else {
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < U.rows) p.y[static_cast<size_t>(U.row0 + t) * p.d + n] = g[t];
        }
      }
    }
    if (!ok) set_abort(C, p.timeouts);
  }
  // The producer and MMA roles run on lane 0 alone: the other lanes wait here for it, so that every
  // warp meets the CTA barrier (and warp 1 the TMEM release) converged.
  __syncwarp();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// Upper bound of the token blocks over all experts (the exact count depends on device offsets).
int ntb_bound(int M_total, int E) { return (M_total + NT - 1) / NT + E; }

size_t counter_bytes(int M_total, int E, int d, int f) {
  const size_t ua = static_cast<size_t>(ntb_bound(M_total, E)) * (f / BM);
  const size_t ub = static_cast<size_t>(ntb_bound(M_total, E)) * (d / BM);
  return ((E + ua + ub) * sizeof(unsigned int) + 255) & ~static_cast<size_t>(255);
}

}  // namespace

size_t grouped_swiglu_dec_tc_workspace(int M_total, int E, int d, int f) {
  const size_t parts = static_cast<size_t>(num_sms()) * 2 * (2 * NT * BM + NT * BM) * sizeof(float);
  return counter_bytes(M_total, E, d, f) + parts;
}

bool grouped_swiglu_dec_tc_supported(int d, int f) {
  return d % KS == 0 && f % KS == 0 && num_sms() <= kMaxCtas &&
         kSmemBytes <= static_cast<size_t>(max_smem_optin());
}

// h: bf16 [M, 2f] (h_hi | h_lo); y_perm: f32 [M, d]; ws: grouped_swiglu_dec_tc_workspace() bytes.
zmoe_status grouped_swiglu_dec_tc(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                                  const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                                  float* y_perm, void* ws, cudaStream_t s) {
  if (!grouped_swiglu_dec_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (decode): needs d % 256 == 0, f % 256 == 0, E <= 64");
  CUtensorMap mg, mu, md, mx, mh;
  bool okm = true;
  {
    // weights viewed as [K/64 chunks][rows][64]: a box of 128 rows x 4 chunks lands as
    // [chunk][row][128 B], the K-major 128-byte-swizzle layout the MMA descriptors describe
    const cuuint64_t dg[3] = {64, static_cast<cuuint64_t>(E) * f, static_cast<cuuint64_t>(d) / 64};
    const cuuint64_t sg[2] = {static_cast<cuuint64_t>(d) * 2, 128};
    const cuuint32_t bw[3] = {64, BM, CH};
    okm = okm && encode_bf16_map(&mg, w_gate, 3, dg, sg, bw) && encode_bf16_map(&mu, w_up, 3, dg, sg, bw);
    const cuuint64_t dd[3] = {64, static_cast<cuuint64_t>(E) * d, static_cast<cuuint64_t>(f) / 64};
    const cuuint64_t sd[2] = {static_cast<cuuint64_t>(f) * 2, 128};
    okm = okm && encode_bf16_map(&md, w_down, 3, dd, sd, bw);
    // token slices: x rows [chunk][16 rows][128 B]; h pair rows [chunk][hi | lo][16 rows][128 B]
    const cuuint64_t dx[3] = {64, static_cast<cuuint64_t>(M_total), static_cast<cuuint64_t>(d) / 64};
    const cuuint64_t sx[2] = {static_cast<cuuint64_t>(d) * 2, 128};
    const cuuint32_t bx[3] = {64, NT, CH};
    okm = okm && encode_bf16_map(&mx, x_perm, 3, dx, sx, bx);
    const cuuint64_t dh[4] = {64, static_cast<cuuint64_t>(M_total), 2, static_cast<cuuint64_t>(f) / 64};
    const cuuint64_t shh[3] = {static_cast<cuuint64_t>(f) * 4, static_cast<cuuint64_t>(f) * 2, 128};
    const cuuint32_t bh[4] = {64, NT, 2, CH};
    okm = okm && encode_bf16_map(&mh, h, 4, dh, shh, bh);
  }
  if (!okm) return fail(ZMOE_ERR_CUDA, "grouped_swiglu (decode): cuTensorMapEncodeTiled failed");
  const int nC = num_sms();
  const size_t ua = static_cast<size_t>(ntb_bound(M_total, E)) * (f / BM);
  const size_t ub = static_cast<size_t>(ntb_bound(M_total, E)) * (d / BM);
  unsigned int* ready = static_cast<unsigned int*>(ws);
  unsigned int* cnt_a = ready + E;
  unsigned int* cnt_b = cnt_a + ua;
  const size_t counters = counter_bytes(M_total, E, d, f);
  float* part_a = reinterpret_cast<float*>(static_cast<unsigned char*>(ws) + counters);
  float* part_b = part_a + static_cast<size_t>(nC) * 2 * 2 * NT * BM;
  if (cudaMemsetAsync(ws, 0, counters, s) != cudaSuccess)
    return check_launch("grouped_swiglu (decode): clearing the counters");
  if (cudaFuncSetAttribute(dec_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSmemBytes)) !=
      cudaSuccess)
    return check_launch("grouped_swiglu (decode): shared memory attribute");
  DecArgs args{offsets, h, y_perm, ready, cnt_a, cnt_b, part_a, part_b, device_timeout_counter(), device_error_counter(),
               E, d, f, M_total, static_cast<int>(ua), static_cast<int>(ub)};
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(nC));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: cut units and phase B wait on others
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, dec_tc_kernel, mg, mu, md, mx, mh, args);
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string("grouped_swiglu (decode): ") + cudaGetErrorString(e));
  return check_launch("grouped_swiglu (decode)");
}

}  // namespace zmoe
