// Decode-size MoE on the tensor cores: the grouped SwiGLU as one swap-AB stream-K launch, and the
// whole MoE layer (pre-norm, router, dispatch, SwiGLU, combine) as one cooperative launch.
//
// Per expert e over its rows of the permuted activations ("GLU Variants Improve Transformer",
// ZONOS2 Technical Report "Builds on"; SiLU per the telknet.cc article on ZONOS2, section 2.1):
//   phase A (gate/up): h = silu(x W_gate[e]^T) * (x W_up[e]^T), stored as the bf16 pair
//                      h_hi = bf16(h), h_lo = bf16(h - h_hi)
//   phase B (down):    y_perm = h_hi W_down[e]^T + h_lo W_down[e]^T          (fp32)
//
// With a few rows per expert the work is streaming the touched experts' weights from HBM once.
// Design of the SwiGLU part:
//   * Swap-AB on tcgen05: 128 weight rows are the MMA's M, a block of up to 16 token rows is its N
//     (kind::f16, bf16 in, fp32 accumulate in TMEM).  A unit is (expert, 128-row weight block, token
//     block); its k-range is cut into 128-wide stages (a 32 KB weight box + a 4 KB x slice or an
//     8 KB h-pair slice).
//   * Stream-K: every CTA (one per SM, cooperative launch: all resident) takes an equal,
//     contiguous range of the stage list of each phase, so bytes per SM balance to within one
//     stage whatever the expert loads are (down to a single expert at batch 1).  A unit wholly
//     inside a CTA's range is finished in TMEM; a unit cut by a range edge leaves fp32 partial
//     sums in a per-CTA slot and the last CTA to arrive adds the partials in CTA order
//     (deterministic) and finishes it.  Each CTA runs its (at most two) cut units first, so the
//     cross-CTA hand-offs overlap the whole units that follow.
//   * Roles: warp 0 loads weight boxes and warp 6 token boxes (x, or the h pair) with TMA into a
//     5-stage ring (200 KB: 160 KB of weights in flight per SM; boxes of 32 KB or more keep one
//     SM's TMA near full HBM rate; 5 x 32 KB measured 2% faster than 2 x 64 KB on the decode step),
//     each completing on its own mbarrier, so weight loads never wait for h; warp 1 allocates TMEM
//     and issues the MMAs from one elected lane (tcgen05.commit frees a stage when its MMAs are
//     done); warps 2..5 read the accumulators with tcgen05.ld and run the epilogues.
//   * fp8 weights (E4M3 codes, one fp32 scale per row): 32 KB boxes of 128 rows x 256 k in a ring of
//     their own; warps 7..10 expand each 128-k half into an f16 A tile in TMEM, the MMAs read A from
//     TMEM, the tokens and the h pair are f16, and the row scales multiply the finished sums.
//   * Phase-A units of expert e release-increment ready[e]; the token producer acquires ready[e]
//     before loading h rows of expert e (cross-proxy fence before the TMA).
//   * Every wait is bounded (time limit): on expiry the CTA counts a device timeout, aborts,
//     drains its own copies and MMAs, frees its TMEM and returns.
//
// The fused layer adds, before the SwiGLU, in the same launch:
//   0a  per token (CTA c takes tokens c, c + C, ...): optional RMSNorm of the fp32 residual stream
//       ("Root Mean Square Layer Normalization", ZONOS2 Technical Report "Builds on"), the router
//       logits, top-k selection on logits + selection bias and the softmax gates (ZONOS2 digest,
//       items 5-6; "Auxiliary-Loss-Free Load Balancing" for the selection-only bias);
//   0b  after a grid barrier, every CTA recomputes the dispatch permutation from all T * k choices
//       (a few hundred integers: cheaper than another barrier) and gathers its share of x_perm;
//   and, after a second barrier, fuses the gate-weighted combine into the down projection's
//   epilogue: y[t] = residual[t] + sum_i gate[t, i] * y_perm[row(t, i)], formed in slot order (for
//   k = 2 by the later of the token's two units, from both rows, so the sum is deterministic).
#include <atomic>

#include "sm100_ptx.cuh"

namespace zmoe {

unsigned int* device_timeout_counter();

namespace {

using namespace ptx;

constexpr int BM = 128;                       // weight rows per unit (MMA M)
constexpr int NT = 16;                        // token rows per block (MMA N)
constexpr int KS = 128;                       // k per stage
constexpr int CH = KS / 64;                   // 64-wide chunks per stage
constexpr int STAGES = 5;
constexpr int W_BYTES = BM * KS * 2;          // 32 KB
constexpr int X_BYTES = NT * KS * 2;          // 4 KB  x slice
constexpr int HP_BYTES = NT * KS * 2 * 2;     // 8 KB  h_hi + h_lo slice
constexpr int kThreads = 224;                 // 7 warps (bf16 weights; fp8 adds 4 converter warps)
constexpr int kMaxWarps = 11;
constexpr int kWarpTok = 6;
constexpr int kWarpConv = 7;                  // fp8: warps 7..10 expand weight boxes to f16
constexpr int KS8 = 256;                      // fp8: k per weight stage (two f16 sub-stages of KS)
constexpr int W8_BYTES = BM * KS8;            // 32 KB of E4M3 codes
constexpr uint32_t TMEM_COLS = 64;            // 2 accumulator buffers x (gate 16 | up 16)
constexpr int kATiles = 4;                    // fp8: f16 A tiles in TMEM (the converters run this far ahead)
constexpr uint32_t TMEM_COLS8 = 512;          // fp8: the accumulators, then kATiles A tiles of 64 columns
constexpr uint32_t kTmemA = 64;               // fp8: first column of A tile 0 (128 k of f16, 2 per column)
static_assert(kTmemA + 64 * kATiles <= TMEM_COLS8, "A tiles must fit in the TMEM allocation");
static_assert(kATiles < STAGES, "an A tile's reuse waits on a token-slot barrier that must not run a phase ahead");
constexpr int kMaxE = 64;
constexpr int kMaxCtas = 256;
constexpr int kMaxAssign = 1024;              // T * k of the fused layer
constexpr unsigned long long kTimeoutNs = 2000000000ull;
constexpr uint32_t kIdesc = idesc_bf16_f32(BM, NT);
// kind::f16 with f16 A and B (format field 0): the fp8 path's expanded weights and f16 tokens.
constexpr uint32_t kIdescF16 = (1u << 4) | (static_cast<uint32_t>(NT >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
constexpr uint32_t kIdesc32 = idesc_bf16_f32(BM, 2 * NT);   // phase B: h_hi and h_lo rows as one operand
constexpr uint32_t kIdescF16x32 =
    (1u << 4) | (static_cast<uint32_t>((2 * NT) >> 3) << 17) | (static_cast<uint32_t>(BM >> 4) << 24);
// fused layer, phase 0 scratch in the (then idle) ring: ids, ranks, the routed row (f32), the raw
// token row, gamma, and the router matrix when it fits.  The bound lies within the ring of either
// weight format (checked in Lay).
constexpr int kRingBytes = 184 * 1024;

constexpr int kScratch0 = 2 * kMaxAssign * 4;

struct DecArgs {
  const int32_t* offsets;   // [E + 1] (grouped-SwiGLU entry; the fused layer forms its own)
  uint16_t* h;              // [M, 2f] h_hi | h_lo
  float* y;                 // [M, d]  y_perm
  unsigned int* ready;      // [E]    finished phase-A units per expert
  unsigned int* cnt_a;      // [ua]   arrivals per cut phase-A unit
  unsigned int* cnt_b;      // [ub]
  float* part_a;            // [C][2 slots][2 mats][NT][BM] partial sums of cut phase-A units
  float* part_b;            // [C][2 slots][NT][BM]
  unsigned int* timeouts;
  unsigned int* errors;
  int E, d, f, M_total;
  int ua_cap, ub_cap;       // units the counter arrays hold
  // combine fused into the phase-B epilogue (fused layer only)
  int fuse, k;
  const float* gates;       // [T, k]
  const float* residual;    // [T, d] or null
  float* out;               // [T, d] (may alias residual)
  unsigned int* comb_cnt;   // [T, d / BM] units of each token's row block done (k = 2)
  // fp8 weights: fp32 scale of each weight row (w = code * scale), applied in the final epilogue
  const float* s_gate;      // [E, f]
  const float* s_up;        // [E, f]
  const float* s_down;      // [E, d]
  // fused layer: x_perm is complete once this counter reaches x_target (grid-wide arrivals)
  const unsigned int* x_ready;
  unsigned int x_target;
  // the phase-A -> phase-B hand-off waits for ready[e] >= (phase-A units of e) + hand_extra, at most
  // hand_limit_ns; hand_extra is 0 except under zmoe_debug_inject_timeout
  unsigned int hand_extra;
  unsigned long long hand_limit_ns;
};

struct LayerArgs {
  const uint16_t* x_in;     // [T, d] layer input (without gamma)
  const float* h_in;        // [T, d] fp32 residual stream, input of the pre-norm (with gamma)
  const float* gamma;       // [d] or null
  float eps;
  const uint16_t* w_r;      // [E, d]
  const float* logit_bias;  // [E] or null
  const float* sel_bias;    // [E] or null
  int T;
  uint16_t* x_norm;         // [T, d] the layer input as routed (written when gamma is given)
  int32_t* expert_idx;      // [T, k]
  float* gates;             // [T, k]
  float* margin;            // [T] or null
  int32_t* counts;          // [E]
  int32_t* offsets;         // [E + 1]
  int32_t* perm;            // [T * k]
  int32_t* inv_perm;        // [T, k]
  uint16_t* x_perm;         // [T * k, d]
  float* logits;            // [T, E] router logits, exchanged through the grid barrier
  unsigned int* gbar;       // grid barrier arrivals
  int G, EG;                // phase-0 items: (token, expert group); EG experts per group
};

struct __align__(16) Ctrl {
  uint64_t full_w[STAGES];
  uint64_t full_t[STAGES];
  uint64_t empty[STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t drain;
  uint64_t rbar[2];          // fused layer: router matrix (+ gamma), token row
  uint64_t tok_empty[STAGES];  // fp8: token slot consumed by the MMAs (bf16: one slot with the weights);
                               // its commit also frees the sub-stage's A tile
  uint64_t afull[kATiles];   // fp8: f16 A tile written to TMEM by the converter warps
  uint32_t tmem_base;
  int abort;
  int bad;
  int last_flag;
  int last_tok[NT];
  int off[kMaxE + 1];
  int ustart[2][kMaxE + 1];  // first unit of each expert, per phase
  int rlo[2][kMaxCtas + 1];  // first stage of each CTA's range, per phase
  // fused layer
  int rowsrc[kMaxAssign];    // permuted row -> token
  int invp[kMaxAssign];      // assignment (t, i) -> permuted row
  float gsm[kMaxAssign];     // gate of assignment (t, i)
  int wcnt[kMaxWarps][kMaxE];
  int run[kMaxE];
  float red[kMaxWarps + 1];
  float wpart[kMaxWarps][16];
  float lbias[kMaxE];        // logit_bias (0 when absent)
  float sbias[kMaxE];        // selection bias (0 when absent)
};

// Shared-memory layout per weight format.  bf16: a ring of STAGES slots, each a 32 KB weight box
// (128 rows x 128 k) and the token slice of the same k.  fp8: a ring of STAGES 32 KB E4M3 boxes
// (128 rows x 256 k) and, apart from it, a ring of STAGES token slices (one per 128 k), so that a
// weight slot is free again as soon as the converter warps have read it.  The control block follows.
template <bool FP8>
struct Lay {
  static constexpr int W_IN = FP8 ? W8_BYTES : W_BYTES;            // bytes of one weight stage
  static constexpr int W_STRIDE = FP8 ? W8_BYTES : W_BYTES + HP_BYTES;
  static constexpr int T_BASE = FP8 ? STAGES * W8_BYTES : W_BYTES;  // token slot 0
  static constexpr int T_STRIDE = FP8 ? HP_BYTES : W_BYTES + HP_BYTES;
  static constexpr int RING = STAGES * (W_IN + HP_BYTES);
  static constexpr int THREADS = FP8 ? kThreads + 128 : kThreads;
  static constexpr int KSTAGE = FP8 ? KS8 : KS;                      // k per weight stage
  static constexpr uint32_t TMEM = FP8 ? TMEM_COLS8 : TMEM_COLS;
  static constexpr size_t SMEM = 1024 + static_cast<size_t>(RING) + sizeof(Ctrl);
  static_assert(W_STRIDE % 1024 == 0 && T_BASE % 1024 == 0 && T_STRIDE % 1024 == 0,
                "swizzled operands need 1024-byte alignment");
  static_assert(SMEM <= 227 * 1024, "ring + control block exceed the 227 KB a B200 CTA may use");
  static_assert(RING >= kRingBytes, "phase-0 scratch must fit in the ring");
};
constexpr size_t kSmemBytes = Lay<false>::SMEM;

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
// shared setup: barriers and TMEM; unit and range tables from C.off
// ------------------------------------------------------------------------------------------
// empty[]: bf16, the MMAs' commit frees the whole slot; fp8, the four converter warps free the weight
// box (tok_empty[] takes the MMAs' commit).
template <bool FP8>
__device__ __forceinline__ void init_ctrl(Ctrl& C) {
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&C.full_w[s], 1);
      mbar_init(&C.full_t[s], 1);
      mbar_init(&C.empty[s], FP8 ? 4 : 1);
      mbar_init(&C.tok_empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&C.tfull[b], 1);
      mbar_init(&C.tempty[b], 4);
    }
    mbar_init(&C.drain, 1);
    mbar_init(&C.rbar[0], 1);
    mbar_init(&C.rbar[1], 1);
    for (int b = 0; b < kATiles; ++b) mbar_init(&C.afull[b], 4);   // one arrival per converter warp
    C.abort = 0;
    C.bad = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if ((threadIdx.x >> 5) == 1) tmem_alloc(&C.tmem_base, Lay<FP8>::TMEM);
}

// Needs C.off; ends with a CTA barrier.  Sets C.bad when the offsets are not a monotone split of
// [0, M_total) or need more units than the counters hold.
__device__ __forceinline__ void build_tables(Ctrl& C, const DecArgs& p, const int* S) {
  const int E = p.E, nC = gridDim.x;
  if (threadIdx.x == 0) {
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
    if (bad) {
      C.bad = 1;
      if (blockIdx.x == 0) record_device_error(p.errors);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i <= nC; i += blockDim.x) {
    C.rlo[0][i] = static_cast<int>(static_cast<long long>(C.ustart[0][E]) * S[0] * i / nC);
    C.rlo[1][i] = static_cast<int>(static_cast<long long>(C.ustart[1][E]) * S[1] * i / nC);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// ------------------------------------------------------------------------------------------
// the SwiGLU roles (both kernels)
// ------------------------------------------------------------------------------------------
// FP8: weight boxes arrive as E4M3 codes (128 rows x 256 k); warps 7..10 expand each 128-k half into an
// f16 A tile in TMEM that the MMAs read, tokens are f16, and the row scales multiply the finished sums.
template <bool FP8>
__device__ __forceinline__ void ffn_roles(const CUtensorMap* mWg, const CUtensorMap* mWu, const CUtensorMap* mWd,
                                          const CUtensorMap* mX, const CUtensorMap* mH, const DecArgs& p, Ctrl& C,
                                          unsigned char* base, uint32_t tmem, const int* S) {
  using LY = Lay<FP8>;
  volatile int* abort_flag = &C.abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = p.E;
  const int nC = gridDim.x, cta = blockIdx.x;

  if (warp == 0 || warp == kWarpTok) {
    // ============================ producers: weights (warp 0), tokens (warp 6) ============================
    if (lane == 0) {
      const bool wt = warp == 0;
      uint64_t* full = wt ? C.full_w : C.full_t;
      // bf16: one token slice per weight stage, in the weight box's slot; fp8: two (one per 128 k of
      // the 256-k box), in the token ring, freed by the MMAs while the converters free the box
      uint64_t* freed = (wt || !FP8) ? C.empty : C.tok_empty;
      const int per = (FP8 && !wt) ? 2 : 1;
      int q = 0;            // loads armed on `full`
      bool ok = true;
      int ready_e = -1;     // last expert whose phase-A units were all seen complete
      if (!wt && p.x_ready) {
        // x_perm is written in this launch by every CTA: wait for all of them (weights need not)
        const uint64_t t0 = globaltimer();
        for (uint32_t it = 0; ld_acquire(p.x_ready) < p.x_target; ++it) {
          if ((it & 15) == 15 && (*abort_flag || globaltimer() - t0 > kTimeoutNs)) {
            ok = false;
            break;
          }
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      for (int ph = 0; ph < 2 && ok; ++ph) {
        const Plan P = make_plan(C.rlo[ph][cta], C.rlo[ph][cta + 1], S[ph]);
        for (int i = 0; i < P.n && ok; ++i) {
          const Seg g = seg_at(P, i);
          const Unit U = unit_of(C, ph, E, g.u);
          for (int j = g.j0; j < g.j1 && ok; ++j) {
            if (!wt && ph == 1 && U.e != ready_e) {
              // every phase-A unit of expert e must have stored its h rows
              const unsigned int target =
                  static_cast<unsigned int>(C.ustart[0][U.e + 1] - C.ustart[0][U.e]) + p.hand_extra;
              const uint64_t t0 = globaltimer();
              for (uint32_t it = 0; ld_acquire(p.ready + U.e) < target; ++it) {
                if ((it & 15) == 15 && (*abort_flag || globaltimer() - t0 > p.hand_limit_ns)) {
                  ok = false;
                  break;
                }
              }
              if (!ok) break;
              ready_e = U.e;
              asm volatile("fence.proxy.async.global;" ::: "memory");
            }
            for (int hs = 0; hs < per; ++hs, ++q) {
              const int slot = q % STAGES;
              const uint32_t epar = static_cast<uint32_t>((q / STAGES) & 1) ^ 1u;
              if (!mbar_wait(&freed[slot], epar, abort_flag, kTimeoutNs)) {
                ok = false;
                break;
              }
              if (wt) {
                unsigned char* dst = base + slot * LY::W_STRIDE;
                mbar_expect_tx(&full[slot], LY::W_IN);
                // bf16: [2 chunks of 64 k][128 rows][128 B]; fp8: [2 chunks of 128 k][128 rows][128 B]
                const int kc = (ph == 0 ? (j >> 1) : j) * CH;
                const CUtensorMap* mw = ph == 1 ? mWd : ((j & 1) ? mWu : mWg);
                tma_load_3d(dst, mw, &full[slot], 0, U.e * (ph == 0 ? p.f : p.d) + U.rb * BM, kc);
              } else {
                unsigned char* dst = base + LY::T_BASE + slot * LY::T_STRIDE;
                // the 128-k block of this slice: the stage's own (bf16), or half hs of the stage (fp8)
                const int kb = (ph == 0 ? (j >> 1) : j) * per + hs;
                if (ph == 0) {
                  mbar_expect_tx(&full[slot], X_BYTES);
                  tma_load_3d(dst, mX, &full[slot], 0, U.row0, kb * CH);
                } else {
                  mbar_expect_tx(&full[slot], HP_BYTES);
                  tma_load_4d(dst, mH, &full[slot], 0, U.row0, 0, kb * CH);
                }
              }
            }
          }
        }
      }
      if (!ok) set_abort(C, p.timeouts);
      if (*abort_flag) drain_ring(full, q);   // no copy may land after the CTA has gone
    }
  } else if (warp == 1) {
    // ===================================== MMA issuer =====================================
    // The whole warp walks the schedule, so that its waits and descriptors stay warp-uniform; one elected
    // lane issues.  An M = 128, N <= 64 MMA costs the issuing thread about as much as it costs the tensor
    // core, so the instruction count is what is kept low: phase B takes h_hi and h_lo as one N = 32
    // operand (its two 16-column halves are summed by the epilogue), and a (sub-)stage ends with a
    // single commit.
    int q = 0;     // bf16: stages consumed; fp8: 128-k sub-stages consumed (two per stage)
    int seg = 0;   // segments (accumulator uses)
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Plan P = make_plan(C.rlo[ph][cta], C.rlo[ph][cta + 1], S[ph]);
      // token operand: phase A the x slice ([chunk][16 rows][128 B]), phase B the h pair ([chunk][32 rows])
      const uint32_t bchunk = static_cast<uint32_t>(ph == 0 ? NT * 128 : 2 * NT * 128);
      const uint32_t idesc = FP8 ? (ph == 0 ? kIdescF16 : kIdescF16x32) : (ph == 0 ? kIdesc : kIdesc32);
      for (int i = 0; i < P.n && ok; ++i) {
        const Seg g = seg_at(P, i);
        const int b = seg & 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&C.tempty[b], static_cast<uint32_t>((seg >> 1) & 1) ^ 1u, abort_flag,
                                               kTimeoutNs));
        if (!ok) break;
        tc_fence_after();
        for (int j = g.j0; j < g.j1 && ok; ++j) {
          // phase A: gate and up stages alternate; the first stage of each matrix in the segment is one of
          // the first two, and its first MMA overwrites that accumulator
          const uint32_t d_tmem = tmem + static_cast<uint32_t>(b * 32 + (ph == 0 ? (j & 1) * 16 : 0));
          const bool fresh = ph == 0 ? j - g.j0 < 2 : j == g.j0;
          for (int hs = 0; hs < (FP8 ? 2 : 1); ++hs, ++q) {
            const int slot = q % STAGES;
            const uint32_t par = static_cast<uint32_t>((q / STAGES) & 1);
            bool got = mbar_wait(FP8 ? &C.afull[q % kATiles] : &C.full_w[slot],
                                 FP8 ? static_cast<uint32_t>((q / kATiles) & 1) : par, abort_flag, kTimeoutNs);
            got = got && mbar_wait(&C.full_t[slot], par, abort_flag, kTimeoutNs);
            ok = __all_sync(0xffffffffu, got);
            if (!ok) break;
            tc_fence_after();
            const uint64_t db = sw128_desc(smem_u32(base + LY::T_BASE + slot * LY::T_STRIDE));
            if (elect_one()) {
              if (FP8) {
                // 16 k per MMA: 8 TMEM columns of the A tile
                const uint32_t ta = tmem + kTmemA + static_cast<uint32_t>((q % kATiles) * 64);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                  umma_tmem_a(d_tmem, ta + static_cast<uint32_t>(kk * 8),
                              db + (((kk >> 2) * bchunk + (kk & 3) * 32) >> 4), idesc,
                              (fresh && hs == 0 && kk == 0) ? 0u : 1u);
                umma_commit(&C.tok_empty[slot]);
              } else {
                const uint64_t da = sw128_desc(smem_u32(base + slot * LY::W_STRIDE));
#pragma unroll
                for (int c = 0; c < CH; ++c)
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk)
                    umma_bf16(d_tmem, da + static_cast<uint64_t>((c * (BM * 128) + kk * 32) >> 4),
                              db + ((c * bchunk + kk * 32) >> 4), idesc, (fresh && c == 0 && kk == 0) ? 0u : 1u);
                umma_commit(&C.empty[slot]);
              }
            }
            __syncwarp();
          }
        }
        if (!ok) break;
        if (elect_one()) umma_commit(&C.tfull[b]);
        __syncwarp();
        ++seg;
      }
    }
    if (!ok && lane == 0) set_abort(C, p.timeouts);
    // every MMA this warp issued completes before the drain barrier flips
    if (elect_one()) umma_commit(&C.drain);
    __syncwarp();
    const uint64_t t1 = globaltimer();
    while (!mbar_try_wait(&C.drain, 0) && globaltimer() - t1 < kTimeoutNs) {
    }
  } else if (warp >= 2 && warp <= 5) {
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
          tmem_ld16(taddr + 16, r1);
          tmem_wait_ld();
          // phase A: gate in columns 0..15, up in 16..31; a segment without gate (up) stages left that
          // accumulator untouched: it contributes 0.  Phase B: W h_hi in columns 0..15, W h_lo in 16..31.
          const bool has_g = ph == 1 || sg.j0 < sg.j1 - 1 || (sg.j0 & 1) == 0;
          const bool has_u = ph == 0 && (sg.j0 < sg.j1 - 1 || (sg.j0 & 1) == 1);
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            const float a0 = __uint_as_float(r0[t]), a1 = __uint_as_float(r1[t]);
            g[t] = ph == 1 ? a0 + a1 : (has_g ? a0 : 0.f);
            v[t] = has_u ? a1 : 0.f;
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
        if (FP8) {
          // w = code * scale: the row's scale multiplies its finished sums
          const float sa = __ldg((ph == 0 ? p.s_gate : p.s_down) + static_cast<size_t>(U.e) * (ph == 0 ? p.f : p.d) + n);
          const float su = ph == 0 ? __ldg(p.s_up + static_cast<size_t>(U.e) * p.f + n) : 1.f;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            g[t] *= sa;
            v[t] *= su;
          }
        }
        if (ph == 0) {
          const size_t ld = static_cast<size_t>(2) * p.f;
#pragma unroll
          for (int t = 0; t < NT; ++t) {
            if (t < U.rows) {
              const float hv = g[t] / (1.f + expf(-g[t])) * v[t];
              uint16_t* hr = p.h + static_cast<size_t>(U.row0 + t) * ld;
              if (FP8) {
                // the f16 pair: the fp8 path's MMAs take f16 operands
                const __half hh = __float2half_rn(hv);
                if (__hisinf(hh)) record_device_error(p.errors);   // |h| beyond the f16 range
                hr[n] = __half_as_ushort(hh);
                hr[p.f + n] = __half_as_ushort(__float2half_rn(hv - __half2float(hh)));
              } else {
                const uint16_t hi = f32_to_bf16_bits(hv);
                hr[n] = hi;
                hr[p.f + n] = f32_to_bf16_bits(hv - bf16_to_f32(hi));
              }
            }
          }
          epi_bar();
          if (et == 0) red_release_add(p.ready + U.e, 1u);
        } else {
#pragma unroll
          for (int t = 0; t < NT; ++t)
            if (t < U.rows) p.y[static_cast<size_t>(U.row0 + t) * p.d + n] = g[t];
          if (p.fuse) {
            if (p.k == 1) {
              // one row per token: y = residual + gate * y_perm, written here
#pragma unroll
              for (int t = 0; t < NT; ++t)
                if (t < U.rows) {
                  const int tok = C.rowsrc[U.row0 + t];
                  const size_t o = static_cast<size_t>(tok) * p.d + n;
                  float acc = fmaf(C.gsm[tok], g[t], 0.f);
                  if (p.residual) acc += p.residual[o];
                  p.out[o] = acc;
                }
            } else {
              // two rows per token, in different units: the later of the two forms the sum from both
              // rows in slot order, so the result does not depend on which unit finished first
              epi_bar();
              if (et < U.rows) {
                const int tok = C.rowsrc[U.row0 + et];
                const int want = (C.invp[2 * tok] >= 0) + (C.invp[2 * tok + 1] >= 0);
                const unsigned int old = atom_acq_rel_add(p.comb_cnt + static_cast<size_t>(tok) * (p.d / BM) + U.rb, 1u);
                C.last_tok[et] = old == static_cast<unsigned int>(want - 1);
              }
              epi_bar();
#pragma unroll
              for (int t = 0; t < NT; ++t)
                if (t < U.rows && C.last_tok[t]) {
                  const int tok = C.rowsrc[U.row0 + t];
                  const size_t o = static_cast<size_t>(tok) * p.d + n;
                  float acc = 0.f;
#pragma unroll
                  for (int s = 0; s < 2; ++s) {
                    const int r = C.invp[2 * tok + s];
                    if (r >= 0) acc = fmaf(C.gsm[2 * tok + s], __ldcg(p.y + static_cast<size_t>(r) * p.d + n), acc);
                  }
                  if (p.residual) acc += p.residual[o];
                  p.out[o] = acc;
                }
            }
          }
        }
      }
    }
    if (!ok) set_abort(C, p.timeouts);
  } else if (FP8 && warp >= kWarpConv) {
    // ===================== fp8 converters (warps 7..10): E4M3 box -> f16 A tile in TMEM =====================
    // A thread expands one weight row, row 32 (warp % 4) + lane: the TMEM lane its warp may write.  For
    // each 128-k half of the 256-k box it reads the row's eight 16-byte units (128-byte swizzle: unit u
    // of row r at u ^ (r % 8), so a quarter-warp's reads hit distinct banks), converts them to 64 f16
    // pairs and stores those into the next of the kATiles A tiles.  Wait outcomes are made warp-uniform:
    // the TMEM stores are warp-collective.
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) + kTmemA;
    int q = 0;   // weight stages
    bool ok = true;
    for (int ph = 0; ph < 2 && ok; ++ph) {
      const Plan P = make_plan(C.rlo[ph][cta], C.rlo[ph][cta + 1], S[ph]);
      for (int i = 0; i < P.n && ok; ++i) {
        const Seg g = seg_at(P, i);
        for (int j = g.j0; j < g.j1 && ok; ++j, ++q) {
          const int slot = q % STAGES;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&C.full_w[slot], static_cast<uint32_t>((q / STAGES) & 1), abort_flag, kTimeoutNs));
          if (!ok) break;
          const unsigned char* box = base + slot * LY::W_STRIDE + r * 128;
          for (int hs = 0; hs < 2 && ok; ++hs) {
            const int q2 = 2 * q + hs, ab = q2 % kATiles;
            // A tile ab last held sub-stage q2 - kATiles: its MMAs are done once that sub-stage's commit (on
            // its token slot) has landed.  That barrier cannot have moved on by a further phase: the next
            // one needs sub-stage q2 - kATiles + STAGES > q2.
            if (q2 >= kATiles) {
              const int prev = q2 - kATiles;
              ok = __all_sync(0xffffffffu, mbar_wait(&C.tok_empty[prev % STAGES],
                                                     static_cast<uint32_t>((prev / STAGES) & 1), abort_flag,
                                                     kTimeoutNs));
              if (!ok) break;
            }
            tc_fence_after();
            const unsigned char* row = box + hs * (BM * 128);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
              uint32_t v[32];
#pragma unroll
              for (int uu = 0; uu < 4; ++uu) {
                const int u = half * 4 + uu;
                const uint4 wv = *reinterpret_cast<const uint4*>(row + ((u ^ (r & 7)) << 4));
                v[uu * 8 + 0] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.x));
                v[uu * 8 + 1] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.x >> 16));
                v[uu * 8 + 2] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.y));
                v[uu * 8 + 3] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.y >> 16));
                v[uu * 8 + 4] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.z));
                v[uu * 8 + 5] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.z >> 16));
                v[uu * 8 + 6] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.w));
                v[uu * 8 + 7] = e4m3x2_to_f16x2(static_cast<uint16_t>(wv.w >> 16));
              }
              tmem_st32(trow + static_cast<uint32_t>(ab * 64 + half * 32), v);
            }
            if (hs == 1) {
              // the whole box is in registers or TMEM: its slot may refill
              __syncwarp();
              if (lane == 0) mbar_arrive(&C.empty[slot]);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&C.afull[ab]);
          }
        }
      }
    }
    if (!ok) set_abort(C, p.timeouts);
  }
}

// ------------------------------------------------------------------------------------------
// kernel 1: the grouped SwiGLU (offsets from the caller)
// ------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(kThreads, 1)
    dec_tc_kernel(const __grid_constant__ CUtensorMap mapWg, const __grid_constant__ CUtensorMap mapWu,
                  const __grid_constant__ CUtensorMap mapWd, const __grid_constant__ CUtensorMap mapX,
                  const __grid_constant__ CUtensorMap mapH, DecArgs p) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctrl& C = *reinterpret_cast<Ctrl*>(base + Lay<false>::RING);
  const int S[2] = {2 * (p.d / KS), p.f / KS};   // stages per unit; phase A alternates gate / up along k
  init_ctrl<false>(C);
  for (int i = threadIdx.x; i <= p.E; i += blockDim.x) C.off[i] = p.offsets[i];
  __syncthreads();
  build_tables(C, p, S);
  const uint32_t tmem = C.tmem_base;
  if (!C.bad) ffn_roles<false>(&mapWg, &mapWu, &mapWd, &mapX, &mapH, p, C, base, tmem, S);
  // The producer and MMA roles run on lane 0 alone: the other lanes wait here for it, so that every
  // warp meets the CTA barrier (and warp 1 the TMEM release) converged.
  __syncwarp();
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

// ------------------------------------------------------------------------------------------
// kernel 2: the fused MoE layer
// ------------------------------------------------------------------------------------------

// Grid-wide barrier over a counter zeroed before the launch: arrival `round` waits for
// round * gridDim.x arrivals (bounded; on expiry the CTA aborts).  False after an abort.
__device__ __forceinline__ bool grid_barrier(unsigned int* ctr, unsigned int round, Ctrl& C, unsigned int* timeouts) {
  __syncthreads();
  if (threadIdx.x == 0) {
    red_release_add(ctr, 1u);
    const unsigned int target = round * gridDim.x;
    const uint64_t t0 = globaltimer();
    for (uint32_t it = 0; ld_acquire(ctr) < target; ++it) {
      if ((it & 15) == 15 && globaltimer() - t0 > kTimeoutNs) {
        set_abort(C, timeouts);
        break;
      }
    }
  }
  __syncthreads();
  return *reinterpret_cast<volatile int*>(&C.abort) == 0;
}

// Phase 0 runs on every warp of the CTA (7 with bf16 weights, 11 with fp8).
__device__ __forceinline__ int nthreads() { return static_cast<int>(blockDim.x); }
__device__ __forceinline__ int nwarps() { return static_cast<int>(blockDim.x >> 5); }

__device__ __forceinline__ float block_sum(float v, Ctrl& C) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) C.red[warp] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
    for (int w = 0; w < nwarps(); ++w) s += C.red[w];
    C.red[nwarps()] = s;
  }
  __syncthreads();
  return C.red[nwarps()];
}

// Phase 0a scratch in the ring (byte offsets; all multiples of 16).
struct RouteSmem {
  float* xs;           // [d]     the routed row, f32 values of the bf16 layer input
  unsigned char* raw;  // [4 d]   the token row as loaded (f32 h or bf16 x)
  float* gam;          // [d]
  uint16_t* wr;        // [EG, d] this CTA's router rows, or null when they do not fit (read from global)
};

__device__ __forceinline__ RouteSmem route_smem(unsigned char* base, int d, int EG) {
  RouteSmem R;
  R.xs = reinterpret_cast<float*>(base + kScratch0);
  R.raw = base + kScratch0 + 4 * d;
  R.gam = reinterpret_cast<float*>(base + kScratch0 + 8 * d);
  const size_t w_off = static_cast<size_t>(kScratch0) + 12 * static_cast<size_t>(d);
  R.wr = (w_off + static_cast<size_t>(EG) * d * 2 <= static_cast<size_t>(kRingBytes))
             ? reinterpret_cast<uint16_t*>(base + w_off)
             : nullptr;
  return R;
}

// Bulk copy of `bytes` (multiple of 16) in pieces of at most 32 KB onto one mbarrier phase.
__device__ __forceinline__ void bulk_load_split(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  for (uint32_t o = 0; o < bytes; o += 32768u) {
    const uint32_t n = bytes - o < 32768u ? bytes - o : 32768u;
    bulk_load(static_cast<unsigned char*>(dst) + o, static_cast<const unsigned char*>(src) + o, n, bar);
  }
}

// Phase 0a item `it` of this CTA: token t, expert group g (experts [g EG, g EG + ne)).  The routed
// input row (RMSNorm'd from h_in when gamma is given, rounded to bf16 like the layer input it stands
// for; group 0 publishes it as x_norm) and its logits for the group's experts, published to
// L.logits.  Thread 0 has this CTA's router rows and gamma in flight on rbar[0] and loads the token
// row onto rbar[1].  False when a wait gave up.
__device__ __forceinline__ bool route_item(const LayerArgs& L, const DecArgs& p, Ctrl& C, const RouteSmem& R, int t,
                                           int g, int it) {
  const int d = p.d, E = p.E;
  const int e0 = g * L.EG;
  const int ne = (E - e0) < L.EG ? (E - e0) : L.EG;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort_flag = &C.abort;
  if (threadIdx.x == 0) {
    // generic reads of the previous row are done (barrier at the end of the last item)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    const uint32_t bytes = static_cast<uint32_t>(d) * (L.gamma ? 4u : 2u);
    mbar_expect_tx(&C.rbar[1], bytes);
    bulk_load_split(R.raw, L.gamma ? static_cast<const void*>(L.h_in + static_cast<size_t>(t) * d)
                                   : static_cast<const void*>(L.x_in + static_cast<size_t>(t) * d),
                    bytes, &C.rbar[1]);
  }
  bool ok = mbar_wait(&C.rbar[1], static_cast<uint32_t>(it & 1), abort_flag, kTimeoutNs);
  if (it == 0 && (L.gamma || (R.wr && L.w_r))) ok = ok && mbar_wait(&C.rbar[0], 0, abort_flag, kTimeoutNs);
  if (!__syncthreads_and(ok)) {
    if (threadIdx.x == 0) set_abort(C, p.timeouts);
    return false;
  }
  if (L.gamma) {
    const float* hr = reinterpret_cast<const float*>(R.raw);
    float ss = 0.f;
    for (int v = threadIdx.x; v < d / 4; v += nthreads()) {
      const float4 a = reinterpret_cast<const float4*>(hr)[v];
      ss += a.x * a.x + a.y * a.y + a.z * a.z + a.w * a.w;
    }
    ss = block_sum(ss, C);
    const float inv = rsqrtf(ss / static_cast<float>(d) + L.eps);
    for (int v = threadIdx.x; v < d / 8; v += nthreads()) {
      // 16-byte shared-memory accesses (a lane's 8 floats are 32 bytes: scalar ones conflict 8 ways)
      const float4 h0 = reinterpret_cast<const float4*>(hr)[2 * v], h1 = reinterpret_cast<const float4*>(hr)[2 * v + 1];
      const float4 g0 = reinterpret_cast<const float4*>(R.gam)[2 * v], g1 = reinterpret_cast<const float4*>(R.gam)[2 * v + 1];
      const float hv[8] = {h0.x, h0.y, h0.z, h0.w, h1.x, h1.y, h1.z, h1.w};
      const float gv[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
      uint16_t b[8];
      float xv[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        b[i] = f32_to_bf16_bits(hv[i] * inv * gv[i]);
        xv[i] = bf16_to_f32(b[i]);
      }
      reinterpret_cast<float4*>(R.xs)[2 * v] = make_float4(xv[0], xv[1], xv[2], xv[3]);
      reinterpret_cast<float4*>(R.xs)[2 * v + 1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
      if (g == 0) {
        uint4 pk;
        pk.x = b[0] | (static_cast<uint32_t>(b[1]) << 16);
        pk.y = b[2] | (static_cast<uint32_t>(b[3]) << 16);
        pk.z = b[4] | (static_cast<uint32_t>(b[5]) << 16);
        pk.w = b[6] | (static_cast<uint32_t>(b[7]) << 16);
        reinterpret_cast<uint4*>(L.x_norm + static_cast<size_t>(t) * d)[v] = pk;
      }
    }
  } else {
    for (int v = threadIdx.x; v < d / 8; v += nthreads())
      unpack_bf16x8(reinterpret_cast<const uint4*>(R.raw)[v], R.xs + 8 * v);
  }
  __syncthreads();
  if (!L.w_r) {
    // no router (E == 1, a dense FFN layer): the single logit is 0 and its gate 1
    if (threadIdx.x == 0) L.logits[static_cast<size_t>(t) * E] = 0.f;
    return true;
  }
  // logits, fp32 accumulation: thread i owns the 8-wide slices i, i + 224, ... of the row and
  // accumulates up to 16 experts on them, then the partial sums are reduced over each warp and
  // across the warps
  for (int j0 = 0; j0 < ne; j0 += 16) {
    float acc[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) acc[j] = 0.f;
    for (int v = threadIdx.x; v < d / 8; v += nthreads()) {
      const float4 xa = reinterpret_cast<const float4*>(R.xs)[2 * v], xb = reinterpret_cast<const float4*>(R.xs)[2 * v + 1];
      const float xv[8] = {xa.x, xa.y, xa.z, xa.w, xb.x, xb.y, xb.z, xb.w};
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (j0 + j < ne) {
          const uint4 w = R.wr ? reinterpret_cast<const uint4*>(R.wr + static_cast<size_t>(j0 + j) * d)[v]
                               : __ldg(reinterpret_cast<const uint4*>(L.w_r + static_cast<size_t>(e0 + j0 + j) * d) + v);
          float wf[8];
          unpack_bf16x8(w, wf);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[j] = fmaf(wf[i], xv[i], acc[j]);
        }
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
    }
    if (lane == 0) {
#pragma unroll
      for (int j = 0; j < 16; ++j) C.wpart[warp][j] = acc[j];
    }
    __syncthreads();
    if (threadIdx.x < 16 && j0 + threadIdx.x < ne) {
      float sum = 0.f;
      for (int w = 0; w < nwarps(); ++w) sum += C.wpart[w][threadIdx.x];
      L.logits[static_cast<size_t>(t) * E + e0 + j0 + threadIdx.x] = sum;
    }
    __syncthreads();
  }
  return true;
}

// Phase 0b (every CTA, one thread per token): top-k of s = q + sel_bias (ties -> lower index) and
// the softmax gates of q = logit + logit_bias, from the published logits.  Writes the choices to
// ids (shared, [T k]) and the gates to C.gsm; CTA 0 also publishes expert_idx, gates and margin.
__device__ __forceinline__ void select_all(const LayerArgs& L, const DecArgs& p, Ctrl& C, int* ids, float* scratch,
                                           size_t scratch_bytes) {
  const int E = p.E, k = p.k;
  const float NEG = -INFINITY;
  // all logits at once (one coalesced pass) when they fit in the scratch, so that the per-token
  // loops below read shared memory instead of issuing dependent global loads
  const size_t nl = static_cast<size_t>(L.T) * E;
  const float* lbase = L.logits;
  if (nl * 4 <= scratch_bytes) {
    for (size_t i = threadIdx.x; i < nl; i += nthreads()) scratch[i] = __ldcg(L.logits + i);
    lbase = scratch;
  }
  for (int e = threadIdx.x; e < E; e += nthreads()) {
    C.lbias[e] = L.logit_bias ? L.logit_bias[e] : 0.f;
    C.sbias[e] = L.sel_bias ? L.sel_bias[e] : 0.f;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < L.T; t += nthreads()) {
    const float* lg = lbase + static_cast<size_t>(t) * E;
    float s1 = NEG, s2 = NEG, s3 = NEG, q1 = NEG, q2 = NEG, m = NEG;
    int e1 = -1, e2 = -1;
    for (int e = 0; e < E; ++e) {
      const float q = lg[e] + C.lbias[e];
      const float sc = q + C.sbias[e];
      m = fmaxf(m, q);
      // strict ">" keeps the lower index on ties (experts arrive in increasing order)
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
    for (int e = 0; e < E; ++e) z += expf(lg[e] + C.lbias[e] - m);
    if (k == 1) {
      const float gt = expf(q1 - m) / z;
      ids[t] = e1;
      C.gsm[t] = gt;
      if (blockIdx.x == 0) {
        L.expert_idx[t] = e1;
        L.gates[t] = gt;
        if (L.margin) L.margin[t] = (E > 1) ? s1 - s2 : INFINITY;
      }
    } else {
      const float z1 = expf(q1 - m), z2 = expf(q2 - m);
      const float inv = 1.f / (z1 + z2);
      ids[2 * t] = e1;
      ids[2 * t + 1] = e2;
      C.gsm[2 * t] = z1 * inv;
      C.gsm[2 * t + 1] = z2 * inv;
      if (blockIdx.x == 0) {
        L.expert_idx[2 * t] = e1;
        L.expert_idx[2 * t + 1] = e2;
        L.gates[2 * t] = z1 * inv;
        L.gates[2 * t + 1] = z2 * inv;
        if (L.margin) L.margin[t] = (E > 2) ? fminf(s1 - s2, s2 - s3) : s1 - s2;
      }
    }
  }
  __syncthreads();
}

__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Phase 0b, after select_all (every CTA, redundantly): counts, offsets and the stable (expert, token)
// order of all T * k assignments in ids into C.off / C.rowsrc / C.invp; CTA 0 publishes them; each
// CTA gathers its share of x_perm.  ids and per-assignment ranks use the (idle) ring as scratch.
__device__ __forceinline__ void permute_all(const LayerArgs& L, const DecArgs& p, Ctrl& C, int* ids, int* rel,
                                            bool to_f16) {
  const int n = L.T * p.k, E = p.E;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x < E) C.run[threadIdx.x] = 0;
  __syncthreads();
  for (int b0 = 0; b0 < n; b0 += nthreads()) {
    for (int i = threadIdx.x; i < nwarps() * kMaxE; i += nthreads()) (&C.wcnt[0][0])[i] = 0;
    __syncthreads();
    const int a = b0 + threadIdx.x;
    const int e = a < n ? ids[a] : -1;
    const unsigned peers = __match_any_sync(0xffffffffu, e);
    const int rank = __popc(peers & lanemask_lt());
    if (e >= 0 && rank == 0) C.wcnt[warp][e] = __popc(peers);
    __syncthreads();
    if (threadIdx.x < E) {
      int r = C.run[threadIdx.x];
      for (int w = 0; w < nwarps(); ++w) {
        const int c = C.wcnt[w][threadIdx.x];
        C.wcnt[w][threadIdx.x] = r;
        r += c;
      }
      C.run[threadIdx.x] = r;
    }
    __syncthreads();
    if (e >= 0) rel[a] = C.wcnt[warp][e] + rank;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    C.off[0] = 0;
    for (int e = 0; e < E; ++e) C.off[e + 1] = C.off[e] + C.run[e];
  }
  __syncthreads();
  for (int a = threadIdx.x; a < n; a += nthreads()) {
    const int e = ids[a];
    if (e >= 0) {
      const int pos = C.off[e] + rel[a];
      C.invp[a] = pos;
      C.rowsrc[pos] = a / p.k;
    } else {
      C.invp[a] = -1;
    }
  }
  __syncthreads();
  const int rows = C.off[E];
  // the routing outputs: by the last CTA, which holds no x_perm row while rows < grid size
  if (blockIdx.x == gridDim.x - 1) {
    for (int i = threadIdx.x; i < E; i += nthreads()) L.counts[i] = C.run[i];
    for (int i = threadIdx.x; i <= E; i += nthreads()) L.offsets[i] = C.off[i];
    for (int i = threadIdx.x; i < rows; i += nthreads()) L.perm[i] = C.rowsrc[i];
    for (int i = threadIdx.x; i < n; i += nthreads()) L.inv_perm[i] = C.invp[i];
  }
  // x_perm rows, one warp per row, one row per CTA before any CTA takes a second: a CTA still gathering
  // when the others start streaming weights sees its loads and stores queue behind theirs
  const uint16_t* xsrc = L.gamma ? L.x_norm : L.x_in;
  const int vecs = p.d / 8;
  for (int r = blockIdx.x + gridDim.x * warp; r < rows; r += gridDim.x * nwarps()) {
    const uint4* s = reinterpret_cast<const uint4*>(xsrc + static_cast<size_t>(C.rowsrc[r]) * p.d);
    uint4* dst = reinterpret_cast<uint4*>(L.x_perm + static_cast<size_t>(r) * p.d);
    for (int v0 = 0; v0 < vecs; v0 += 32 * 8) {
      uint4 buf[8];   // eight loads in flight per lane
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v0 + j * 32 + lane < vecs) buf[j] = __ldcg(s + v0 + j * 32 + lane);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (v0 + j * 32 + lane < vecs) {
          if (to_f16) {
            // fp8 weights: the MMA operands are f16 (exact for bf16 values in f16's normal range)
            float f8[8];
            unpack_bf16x8(buf[j], f8);
            uint32_t w[4];
            bool inf = false;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const __half2 h2 = __floats2half2_rn(f8[2 * i], f8[2 * i + 1]);
              inf |= __hisinf(__low2half(h2)) || __hisinf(__high2half(h2));
              w[i] = *reinterpret_cast<const uint32_t*>(&h2);
            }
            if (inf) record_device_error(p.errors);
            buf[j] = make_uint4(w[0], w[1], w[2], w[3]);
          }
          dst[v0 + j * 32 + lane] = buf[j];
        }
    }
  }
}

template <bool FP8>
__global__ void __launch_bounds__(Lay<FP8>::THREADS, 1)
    moe_layer_kernel(const __grid_constant__ CUtensorMap mapWg, const __grid_constant__ CUtensorMap mapWu,
                     const __grid_constant__ CUtensorMap mapWd, const __grid_constant__ CUtensorMap mapX,
                     const __grid_constant__ CUtensorMap mapH, DecArgs p, LayerArgs L) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* base =
      reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  Ctrl& C = *reinterpret_cast<Ctrl*>(base + Lay<FP8>::RING);
  // stages per unit (phase A alternates gate / up along k)
  const int S[2] = {2 * (p.d / Lay<FP8>::KSTAGE), p.f / Lay<FP8>::KSTAGE};
  init_ctrl<FP8>(C);
  __syncthreads();
  // the ring is idle until the SwiGLU roles start: phase 0 keeps its scratch there
  int* ids = reinterpret_cast<int*>(base);
  int* rel = ids + kMaxAssign;
  const RouteSmem R = route_smem(base, p.d, L.EG);
  // this CTA's items (t, g) = (i / G, i % G) for i = blockIdx.x, blockIdx.x + C, ...; with G > 1
  // there is at most one item per CTA, so the router rows of one group serve all of them
  const int g0 = static_cast<int>(blockIdx.x) % L.G;
  const int ne0 = (p.E - g0 * L.EG) < L.EG ? (p.E - g0 * L.EG) : L.EG;
  const uint32_t wb = (R.wr && L.w_r) ? static_cast<uint32_t>(ne0) * p.d * 2u : 0u;
  const uint32_t gb = L.gamma ? static_cast<uint32_t>(p.d) * 4u : 0u;
  const bool armed0 = static_cast<int>(blockIdx.x) < L.T * L.G && wb + gb > 0;
  if (threadIdx.x == 0 && armed0) {
    // the router rows (when they fit) and gamma, once per CTA, with the TMA engine: one SM's plain
    // loads keep too few bytes in flight to fetch tens of KB quickly
    mbar_expect_tx(&C.rbar[0], wb + gb);
    if (wb) bulk_load_split(R.wr, L.w_r + static_cast<size_t>(g0) * L.EG * p.d, wb, &C.rbar[0]);
    if (gb) bulk_load_split(R.gam, L.gamma, gb, &C.rbar[0]);
  }
  bool ok = true;
  int nrow = 0;   // token rows loaded onto rbar[1]
  for (int i = blockIdx.x; i < L.T * L.G && ok; i += gridDim.x) ok = route_item(L, p, C, R, i / L.G, i % L.G, nrow++);
  if (!ok && threadIdx.x == 0) {
    // bulk copies that may still be landing in the ring must finish before the CTA moves on
    const uint64_t t1 = globaltimer();
    while (((armed0 && !mbar_try_wait(&C.rbar[0], 0)) ||
            (nrow > 0 && !mbar_try_wait(&C.rbar[1], static_cast<uint32_t>((nrow - 1) & 1)))) &&
           globaltimer() - t1 < kTimeoutNs) {
    }
  }
  if (grid_barrier(L.gbar, 1, C, p.timeouts)) {
    select_all(L, p, C, ids, reinterpret_cast<float*>(base + kScratch0), kRingBytes - kScratch0);
    permute_all(L, p, C, ids, rel, FP8);
    // generic-proxy writes to the ring are ordered before the TMA writes that will reuse it
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    build_tables(C, p, S);   // ends with a CTA barrier: this CTA's x_perm rows are written
    // second grid arrival: x_perm complete here.  Only the token producer waits for all CTAs
    // (DecArgs::x_ready); the weight producer starts streaming at once.  An epilogue thread arrives
    // (its release fence waits for this CTA's gather stores; the producers must not wait on it).
    if (threadIdx.x == 64) red_release_add(L.gbar, 1u);
    if (!C.bad) ffn_roles<FP8>(&mapWg, &mapWu, &mapWd, &mapX, &mapH, p, C, base, C.tmem_base, S);
  }
  __syncwarp();
  __syncthreads();
  if ((threadIdx.x >> 5) == 1) {
    tc_fence_after();
    tmem_dealloc(C.tmem_base, Lay<FP8>::TMEM);
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------

// Upper bound of the token blocks over all experts (the exact count depends on device offsets).
int ntb_bound(int M_total, int E) { return (M_total + NT - 1) / NT + E; }

size_t align256(size_t b) { return (b + 255) & ~static_cast<size_t>(255); }

struct Layout {
  size_t ready, cnt_a, cnt_b, comb, gbar, counters_end;   // counters (one memset)
  size_t part_a, part_b;
  size_t total;
  int ua, ub;
};

// Counters first (zeroed per call), then the per-CTA partial slots.
Layout ffn_layout(int M_total, int E, int d, int f, int T_comb) {
  Layout Lo{};
  Lo.ua = ntb_bound(M_total, E) * (f / BM);
  Lo.ub = ntb_bound(M_total, E) * (d / BM);
  size_t o = 0;
  Lo.ready = o;
  o += static_cast<size_t>(E) * 4;
  Lo.cnt_a = o;
  o += static_cast<size_t>(Lo.ua) * 4;
  Lo.cnt_b = o;
  o += static_cast<size_t>(Lo.ub) * 4;
  Lo.comb = o;
  o += static_cast<size_t>(T_comb) * (d / BM) * 4;
  Lo.gbar = o;
  o += 4;
  Lo.counters_end = align256(o);
  Lo.part_a = Lo.counters_end;
  Lo.part_b = Lo.part_a + static_cast<size_t>(num_sms()) * 2 * 2 * NT * BM * 4;
  Lo.total = Lo.part_b + static_cast<size_t>(num_sms()) * 2 * NT * BM * 4;
  return Lo;
}

struct Maps {
  CUtensorMap g, u, dn, x, h;
};

bool encode_maps(Maps* m, const uint16_t* x_perm, int M_total, const uint16_t* w_gate, const uint16_t* w_up,
                 const uint16_t* w_down, int E, int d, int f, const uint16_t* h) {
  // weights viewed as [K/64 chunks][rows][64]: a box of 128 rows x 4 chunks lands as
  // [chunk][row][128 B], the K-major 128-byte-swizzle layout the MMA descriptors describe
  const cuuint64_t dg[3] = {64, static_cast<cuuint64_t>(E) * f, static_cast<cuuint64_t>(d) / 64};
  const cuuint64_t sg[2] = {static_cast<cuuint64_t>(d) * 2, 128};
  const cuuint32_t bw[3] = {64, BM, CH};
  const cuuint64_t dd[3] = {64, static_cast<cuuint64_t>(E) * d, static_cast<cuuint64_t>(f) / 64};
  const cuuint64_t sd[2] = {static_cast<cuuint64_t>(f) * 2, 128};
  // token slices: x rows [chunk][16 rows][128 B]; h pair rows [chunk][hi | lo][16 rows][128 B]
  const cuuint64_t dx[3] = {64, static_cast<cuuint64_t>(M_total), static_cast<cuuint64_t>(d) / 64};
  const cuuint64_t sx[2] = {static_cast<cuuint64_t>(d) * 2, 128};
  const cuuint32_t bx[3] = {64, NT, CH};
  const cuuint64_t dh[4] = {64, static_cast<cuuint64_t>(M_total), 2, static_cast<cuuint64_t>(f) / 64};
  const cuuint64_t shh[3] = {static_cast<cuuint64_t>(f) * 4, static_cast<cuuint64_t>(f) * 2, 128};
  const cuuint32_t bh[4] = {64, NT, 2, CH};
  return encode_bf16_map(&m->g, w_gate, 3, dg, sg, bw) && encode_bf16_map(&m->u, w_up, 3, dg, sg, bw) &&
         encode_bf16_map(&m->dn, w_down, 3, dd, sd, bw) && encode_bf16_map(&m->x, x_perm, 3, dx, sx, bx) &&
         encode_bf16_map(&m->h, h, 4, dh, shh, bh);
}

template <typename K, typename... Args>
zmoe_status launch_coop(K kernel, const char* what, cudaStream_t s, int threads, size_t smem, Args... args) {
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)) !=
      cudaSuccess)
    return check_launch(what);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(num_sms()));
  cfg.blockDim = dim3(static_cast<unsigned>(threads));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;   // every CTA resident: CTAs wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, args...);
  if (e != cudaSuccess) return fail(ZMOE_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
  return check_launch(what);
}

// Fault injection for tests of the timeout path (zmoe_debug_inject_timeout): host-side settings that
// every launch copies into its arguments.
std::atomic<unsigned int> g_inject_extra{0};
std::atomic<unsigned long long> g_inject_limit_ns{0};

DecArgs dec_args(const Layout& Lo, void* ws, const int32_t* offsets, uint16_t* h, float* y_perm, int E, int d, int f,
                 int M_total) {
  unsigned char* w = static_cast<unsigned char*>(ws);
  DecArgs a{};
  a.offsets = offsets;
  a.h = h;
  a.y = y_perm;
  a.ready = reinterpret_cast<unsigned int*>(w + Lo.ready);
  a.cnt_a = reinterpret_cast<unsigned int*>(w + Lo.cnt_a);
  a.cnt_b = reinterpret_cast<unsigned int*>(w + Lo.cnt_b);
  a.part_a = reinterpret_cast<float*>(w + Lo.part_a);
  a.part_b = reinterpret_cast<float*>(w + Lo.part_b);
  a.timeouts = device_timeout_counter();
  a.errors = device_error_counter();
  a.E = E;
  a.d = d;
  a.f = f;
  a.M_total = M_total;
  a.ua_cap = Lo.ua;
  a.ub_cap = Lo.ub;
  a.hand_extra = g_inject_extra.load();
  a.hand_limit_ns = a.hand_extra ? g_inject_limit_ns.load() : kTimeoutNs;
  return a;
}

}  // namespace

bool grouped_swiglu_dec_tc_supported(int d, int f) {
  return d % KS == 0 && f % KS == 0 && num_sms() <= kMaxCtas && kSmemBytes <= static_cast<size_t>(max_smem_optin());
}

size_t grouped_swiglu_dec_tc_workspace(int M_total, int E, int d, int f) {
  return ffn_layout(M_total, E, d, f, 0).total;
}

// h: bf16 [M, 2f] (h_hi | h_lo); y_perm: f32 [M, d]; ws: grouped_swiglu_dec_tc_workspace() bytes.
zmoe_status grouped_swiglu_dec_tc(const uint16_t* x_perm, const int32_t* offsets, int M_total, const uint16_t* w_gate,
                                  const uint16_t* w_up, const uint16_t* w_down, int E, int d, int f, uint16_t* h,
                                  float* y_perm, void* ws, cudaStream_t s) {
  if (!grouped_swiglu_dec_tc_supported(d, f) || E > kMaxE)
    return fail(ZMOE_ERR_UNSUPPORTED, "grouped_swiglu (decode): needs d % 256 == 0, f % 256 == 0, E <= 64");
  Maps m;
  if (!encode_maps(&m, x_perm, M_total, w_gate, w_up, w_down, E, d, f, h))
    return fail(ZMOE_ERR_CUDA, "grouped_swiglu (decode): cuTensorMapEncodeTiled failed");
  const Layout Lo = ffn_layout(M_total, E, d, f, 0);
  if (cudaMemsetAsync(ws, 0, Lo.counters_end, s) != cudaSuccess)
    return check_launch("grouped_swiglu (decode): clearing the counters");
  const DecArgs args = dec_args(Lo, ws, offsets, h, y_perm, E, d, f, M_total);
  return launch_coop(dec_tc_kernel, "grouped_swiglu (decode)", s, kThreads, kSmemBytes, m.g, m.u, m.dn, m.x, m.h,
                     args);
}

// ------------------------------------------------------------------------------------------
// the fused layer: workspace carve-up and launch
// ------------------------------------------------------------------------------------------
bool moe_layer_fused_supported(int T, int E, int d, int f, int k) {
  return grouped_swiglu_dec_tc_supported(d, f) && E <= kMaxE && T >= 1 && static_cast<long long>(T) * k <= kMaxAssign &&
         static_cast<long long>(kScratch0) + 12LL * d <= kRingBytes;
}

struct LayerWs {
  Layout ffn;
  size_t x_norm, x_perm, h, y_perm, idx, gates, margin, counts, offsets, perm, inv_perm, logits, total;
};

LayerWs layer_ws(int T, int E, int d, int f, int k) {
  LayerWs W{};
  const int n = T * k;
  W.ffn = ffn_layout(n, E, d, f, T);
  size_t o = align256(W.ffn.total);
  auto take = [&o](size_t bytes) {
    const size_t at = o;
    o = align256(o + bytes);
    return at;
  };
  W.x_norm = take(static_cast<size_t>(T) * d * 2);
  W.x_perm = take(static_cast<size_t>(n) * d * 2);
  W.h = take(static_cast<size_t>(n) * 2 * f * 2);
  W.y_perm = take(static_cast<size_t>(n) * d * 4);
  W.idx = take(static_cast<size_t>(n) * 4);
  W.gates = take(static_cast<size_t>(n) * 4);
  W.margin = take(static_cast<size_t>(T) * 4);
  W.counts = take(static_cast<size_t>(E) * 4);
  W.offsets = take(static_cast<size_t>(E + 1) * 4);
  W.perm = take(static_cast<size_t>(n) * 4);
  W.inv_perm = take(static_cast<size_t>(n) * 4);
  W.logits = take(static_cast<size_t>(T) * E * 4);
  W.total = o;
  return W;
}

size_t moe_layer_fused_workspace(int T, int E, int d, int f, int k) { return layer_ws(T, E, d, f, k).total; }

// fp8 weights when s_gate is given: w_gate / w_up / w_down are E4M3 codes with row scales s_*.
zmoe_status moe_layer_fused(const uint16_t* x, const float* h_in, const float* gamma, float eps, const uint16_t* w_r,
                            const float* logit_bias, const float* sel_bias, const void* w_gate, const void* w_up,
                            const void* w_down, int T, int d, int f, int E, int k, float* y, int32_t* expert_idx,
                            float* gates, float* margin, uint16_t* x_norm_out, void* ws, cudaStream_t s,
                            const float* s_gate, const float* s_up, const float* s_down) {
  const bool fp8 = s_gate != nullptr;
  const LayerWs W = layer_ws(T, E, d, f, k);
  unsigned char* w = static_cast<unsigned char*>(ws);
  const int n = T * k;
  uint16_t* xn = x_norm_out ? x_norm_out : reinterpret_cast<uint16_t*>(w + W.x_norm);
  uint16_t* xp = reinterpret_cast<uint16_t*>(w + W.x_perm);
  uint16_t* hh = reinterpret_cast<uint16_t*>(w + W.h);
  float* yp = reinterpret_cast<float*>(w + W.y_perm);
  Maps m;
  bool okm = encode_maps(&m, xp, n, static_cast<const uint16_t*>(w_gate), static_cast<const uint16_t*>(w_up),
                         static_cast<const uint16_t*>(w_down), E, d, f, hh);
  if (okm && fp8) {
    // E4M3 codes viewed as [K/128 chunks][rows][128]: a box of 128 rows x 2 chunks (256 k, 32 KB) lands
    // as [chunk][row][128 B] in the 128-byte swizzle, the layout the converter warps read
    const cuuint64_t dg[3] = {128, static_cast<cuuint64_t>(E) * f, static_cast<cuuint64_t>(d) / 128};
    const cuuint64_t sg[2] = {static_cast<cuuint64_t>(d), 128};
    const cuuint64_t dd[3] = {128, static_cast<cuuint64_t>(E) * d, static_cast<cuuint64_t>(f) / 128};
    const cuuint64_t sd[2] = {static_cast<cuuint64_t>(f), 128};
    const cuuint32_t box[3] = {128, BM, KS8 / 128};
    okm = encode_map(&m.g, w_gate, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, dg, sg, box, CU_TENSOR_MAP_SWIZZLE_128B) &&
          encode_map(&m.u, w_up, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, dg, sg, box, CU_TENSOR_MAP_SWIZZLE_128B) &&
          encode_map(&m.dn, w_down, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, dd, sd, box, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  if (!okm) return fail(ZMOE_ERR_CUDA, "zmoe_moe_layer: cuTensorMapEncodeTiled failed");
  if (cudaMemsetAsync(ws, 0, W.ffn.counters_end, s) != cudaSuccess)
    return check_launch("zmoe_moe_layer: clearing the counters");
  DecArgs a = dec_args(W.ffn, ws, nullptr, hh, yp, E, d, f, n);
  LayerArgs L{};
  L.x_in = x;
  L.h_in = h_in;
  L.gamma = gamma;
  L.eps = eps;
  L.w_r = w_r;
  L.logit_bias = logit_bias;
  L.sel_bias = sel_bias;
  L.T = T;
  L.x_norm = xn;
  L.expert_idx = expert_idx ? expert_idx : reinterpret_cast<int32_t*>(w + W.idx);
  L.gates = gates ? gates : reinterpret_cast<float*>(w + W.gates);
  L.margin = margin;
  L.counts = reinterpret_cast<int32_t*>(w + W.counts);
  L.offsets = reinterpret_cast<int32_t*>(w + W.offsets);
  L.perm = reinterpret_cast<int32_t*>(w + W.perm);
  L.inv_perm = reinterpret_cast<int32_t*>(w + W.inv_perm);
  L.x_perm = xp;
  L.gbar = reinterpret_cast<unsigned int*>(w + W.ffn.gbar);
  L.logits = reinterpret_cast<float*>(w + W.logits);
  // phase-0 items (token, expert group): as many groups as keep every SM busy, up to one per expert
  {
    const int nC = num_sms();
    int G = nC / T;
    G = G < 1 ? 1 : (G > E ? E : G);
    L.EG = (E + G - 1) / G;
    L.G = (E + L.EG - 1) / L.EG;
  }
  a.fuse = 1;
  a.k = k;
  a.gates = L.gates;
  a.residual = h_in;
  a.out = y;
  a.comb_cnt = reinterpret_cast<unsigned int*>(w + W.ffn.comb);
  a.x_ready = L.gbar;                                  // second grid arrival: x_perm complete
  a.x_target = 2u * static_cast<unsigned int>(num_sms());
  a.s_gate = s_gate;
  a.s_up = s_up;
  a.s_down = s_down;
  if (fp8)
    return launch_coop(moe_layer_kernel<true>, "zmoe_moe_layer_fp8 (fused decode)", s, Lay<true>::THREADS,
                       Lay<true>::SMEM, m.g, m.u, m.dn, m.x, m.h, a, L);
  return launch_coop(moe_layer_kernel<false>, "zmoe_moe_layer (fused decode)", s, Lay<false>::THREADS,
                     Lay<false>::SMEM, m.g, m.u, m.dn, m.x, m.h, a, L);
}

}  // namespace zmoe

extern "C" zmoe_status zmoe_debug_inject_timeout(uint32_t extra, uint64_t limit_ns) {
  ZMOE_REQUIRE(extra == 0 || (limit_ns >= 1000ull && limit_ns <= 2000000000ull),
               "zmoe_debug_inject_timeout: limit_ns must be in [1 us, 2 s] when extra > 0");
  zmoe::clear_error();
  zmoe::g_inject_limit_ns.store(extra ? limit_ns : 0ull);
  zmoe::g_inject_extra.store(extra);
  return ZMOE_OK;
}
