"""Seeded synthetic inputs for the sparse MoE feed-forward path.

This module is shared by the fp64 oracle (``oracle/``) and by the CUDA path's
tests and benchmark.  It only draws random numbers and stores them; it holds
none of the method's arithmetic (no routing, no normalisation, no FFN).

Conventions
-----------
* Generator: ``numpy.random.default_rng(seed)`` (PCG64), seed 0 unless stated.
* Draw order inside one layer: x, W_r, W_gate, W_up, W_down, b, logit_bias,
  gamma.  Expert tensors are drawn as one ``[E, ...]`` array, i.e. in expert
  order.
* ``N(mu, v)``: the second argument is the VARIANCE (so ``N(0, 1/fan_in)``
  has standard deviation ``1/sqrt(fan_in)``).
* bf16 configurations: every floating value is drawn in fp32 and rounded to
  the nearest bf16 (ties to even).  The arrays handed out are float32 arrays
  whose values are exactly representable in bf16, so the GPU side converts
  them without loss and the oracle reads them exactly in fp64.
* Expert weights are row-major and K-major: ``W_gate, W_up: [E, f, d]``,
  ``W_down: [E, d, f]``, router ``W_r: [E, d]``.

The five workloads are the ones the ZONOS2 pages describe the MoE decoder
with (ZONOS2 Technical Report digest, "method overview and architecture",
item 5: 16 experts, top-1 routing, top-2 in the last MoE layer; item 1: nine
delay-patterned DAC codebooks), at d_model = 2048 and d_ff = 3072.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

NUM_CODEBOOKS = 9          # N: DAC residual codebooks per frame
CODEBOOK_SIZE = 1024       # ids 0..1023
PAD_ID = 1024              # pad id used outside the delay pattern's valid range
VOCAB_ROWS = CODEBOOK_SIZE + 1   # V: embedding rows per codebook table (pad row included)

D_MODEL = 2048
D_FF = 3072
NUM_EXPERTS = 16
NUM_MOE_LAYERS = 24


def round_to_bf16(a: np.ndarray, inplace: bool = False) -> np.ndarray:
    """Round a float32 array to the nearest bf16 value (ties to even).

    Returns float32 values that are exactly representable in bf16.  (Finite
    inputs below the largest bf16 only; random draws here never come close.)
    Works in place, chunk by chunk, when ``inplace`` is set and ``a`` is a
    contiguous float32 array.
    """
    if not (inplace and isinstance(a, np.ndarray) and a.dtype == np.float32 and a.flags.c_contiguous):
        a = np.array(a, dtype=np.float32, copy=True, order="C")
    u = a.reshape(-1).view(np.uint32)
    chunk = 1 << 20
    lsb = np.empty(min(chunk, u.size), np.uint32)
    for lo in range(0, u.size, chunk):
        c = u[lo:lo + chunk]
        t = lsb[:c.size]
        np.right_shift(c, np.uint32(16), out=t)
        t &= np.uint32(1)
        t += np.uint32(0x7FFF)
        c += t
        c &= np.uint32(0xFFFF0000)
    return a


def quantize_e4m3_rows(w: np.ndarray):
    """Weights stored as fp8: per output row (last axis = the contraction), scale = max|w| / 448 and
    codes = the E4M3 (bias 7, no infinities, largest finite 448) value nearest w / scale, ties to even.

    Returns (codes uint8 of w's shape, scales float32 of w.shape[:-1]).  This is the storage format the
    fp8 path reads (a checkpoint would hold it); both the GPU and the oracle consume these arrays.
    """
    w = np.asarray(w, np.float32)
    amax = np.max(np.abs(w), axis=-1)
    scales = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    v = (w / scales[..., None]).astype(np.float64)
    a = np.abs(v)
    # binade of each value (subnormals share the lowest normal binade's spacing, 2^-9)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.clip(e, -6, 8)
    ulp = np.exp2(e - 3)
    q = np.round(a / ulp) * ulp                 # numpy rounds half to even
    q = np.minimum(q, 448.0)
    # encode: exponent field and 3 mantissa bits (subnormals: exponent field 0)
    eq = np.floor(np.log2(np.where(q > 0, q, 1.0)))
    normal = (q >= 2.0 ** -6)
    efield = np.where(normal, eq + 7, 0).astype(np.int64)
    mant = np.where(normal, np.round((q / np.exp2(eq) - 1.0) * 8), np.round(q / 2.0 ** -9)).astype(np.int64)
    codes = ((efield << 3) | mant) & 0x7F
    codes = np.where(q == 0, 0, codes) | np.where(v < 0, 0x80, 0)
    return codes.astype(np.uint8), scales


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """The bf16 bit patterns (uint16) of a float32 array already rounded to bf16."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def _normal(rng: np.random.Generator, shape, var: float, bf16: bool) -> np.ndarray:
    out = rng.standard_normal(size=shape, dtype=np.float32)
    if var != 1.0:
        out *= np.float32(np.sqrt(var))
    return round_to_bf16(out, inplace=True) if bf16 else out


def zipf_logit_bias(num_experts: int, s: float) -> np.ndarray:
    """log p_e with p_e proportional to (e+1)^-s: expert 0 is the heaviest."""
    w = np.arange(1, num_experts + 1, dtype=np.float64) ** (-s)
    return np.log(w / w.sum()).astype(np.float32)


@dataclass
class MoELayerInputs:
    """One MoE layer's inputs and weights (float32 arrays; bf16-exact when dtype == 'bf16')."""

    dtype: str                 # 'f32' or 'bf16'
    k: int                     # experts per token
    x: np.ndarray              # [T, d]
    w_router: np.ndarray       # [E, d]
    w_gate: np.ndarray         # [E, f, d]
    w_up: np.ndarray           # [E, f, d]
    w_down: np.ndarray         # [E, d, f]
    sel_bias: np.ndarray       # [E] float32, selection-only bias b_l
    logit_bias: Optional[np.ndarray] = None   # [E] float32 or None
    gamma: Optional[np.ndarray] = None        # [d] float32 (per-layer RMSNorm gain, stack only)
    meta: dict = field(default_factory=dict)

    @property
    def T(self) -> int:
        return self.x.shape[0]

    @property
    def d(self) -> int:
        return self.x.shape[1]

    @property
    def E(self) -> int:
        return self.w_router.shape[0]

    @property
    def f(self) -> int:
        return self.w_gate.shape[1]


def make_moe_layer(T: int, d: int, f: int, E: int, k: int, dtype: str = "bf16", seed: int = 0,
                   sel_bias_var: float = 0.0, zipf_s: Optional[float] = None,
                   x_var: float = 1.0, with_gamma: bool = False,
                   draw_x: bool = True) -> MoELayerInputs:
    """Draw one MoE layer in the documented order.

    x ~ N(0, x_var); W_r, W_gate, W_up ~ N(0, 1/d); W_down ~ N(0, 1/f);
    b ~ N(0, sel_bias_var) (zeros when 0); logit_bias = log Zipf(zipf_s) or None;
    gamma ~ N(1, 0.01) when requested.
    """
    if dtype not in ("f32", "bf16"):
        raise ValueError(f"dtype must be 'f32' or 'bf16', got {dtype!r}")
    bf = dtype == "bf16"
    rng = np.random.default_rng(seed)
    x = _normal(rng, (T, d), x_var, bf) if draw_x else np.zeros((T, d), np.float32)
    w_router = _normal(rng, (E, d), 1.0 / d, bf)
    w_gate = _normal(rng, (E, f, d), 1.0 / d, bf)
    w_up = _normal(rng, (E, f, d), 1.0 / d, bf)
    w_down = _normal(rng, (E, d, f), 1.0 / f, bf)
    if sel_bias_var > 0.0:
        sel_bias = rng.standard_normal(E, dtype=np.float32) * np.float32(np.sqrt(sel_bias_var))
    else:
        sel_bias = np.zeros(E, np.float32)
    logit_bias = zipf_logit_bias(E, zipf_s) if zipf_s is not None else None
    gamma = None
    if with_gamma:
        gamma = (1.0 + 0.1 * rng.standard_normal(d, dtype=np.float32)).astype(np.float32)
    return MoELayerInputs(dtype=dtype, k=k, x=x, w_router=w_router, w_gate=w_gate, w_up=w_up,
                          w_down=w_down, sel_bias=sel_bias.astype(np.float32), logit_bias=logit_bias,
                          gamma=gamma, meta=dict(seed=seed, sel_bias_var=sel_bias_var, zipf_s=zipf_s))


def make_codes(frames: int, num_codebooks: int = NUM_CODEBOOKS, seed: int = 0,
               batch: Optional[int] = None) -> np.ndarray:
    """Codebook ids uniform in [0, CODEBOOK_SIZE): int32 [frames, N] or [batch, frames, N]."""
    rng = np.random.default_rng(seed)
    shape = (frames, num_codebooks) if batch is None else (batch, frames, num_codebooks)
    return rng.integers(0, CODEBOOK_SIZE, size=shape, dtype=np.int64).astype(np.int32)


# --------------------------------------------------------------------------------------------
# The five workloads.
# --------------------------------------------------------------------------------------------

CONFIG_NAMES = {
    1: "tiny MoE layer fp32 (T=64, d=128, f=256, E=4, top-1) + delay shear of int32[16,9]",
    2: "decode step, one MoE layer bf16 (T=64, d=2048, f=3072, E=16, top-1)",
    3: "prefill MoE layer bf16 (T=16384, d=2048, f=3072, E=16, top-1, b~N(0,0.5))",
    4: "final MoE layer bf16 (T=16384, d=2048, f=3072, E=16, top-2, Zipf(1.2) logit skew)",
    5: "batch-1 decode stack bf16 (embed-sum + RMSNorm, 24 MoE layers, top-2 in the last)",
}


def make_config(cfg: int, seed: int = 0, T: Optional[int] = None) -> MoELayerInputs:
    """The layer of configuration ``cfg`` (1..4).  ``T`` overrides the token count."""
    if cfg == 1:
        return make_moe_layer(T or 64, 128, 256, 4, 1, "f32", seed)
    if cfg == 2:
        return make_moe_layer(T or 64, D_MODEL, D_FF, NUM_EXPERTS, 1, "bf16", seed, sel_bias_var=0.1)
    if cfg == 3:
        return make_moe_layer(T or 16384, D_MODEL, D_FF, NUM_EXPERTS, 1, "bf16", seed, sel_bias_var=0.5)
    if cfg == 4:
        return make_moe_layer(T or 16384, D_MODEL, D_FF, NUM_EXPERTS, 2, "bf16", seed, zipf_s=1.2)
    raise ValueError(f"config {cfg} is not a single-layer configuration")


def config1_codes(seed: int = 0) -> np.ndarray:
    """The delay-pattern input of configuration 1: int32 [16 frames, 9 codebooks]."""
    return make_codes(16, NUM_CODEBOOKS, seed)


# --------------------------------------------------------------------------------------------
# Configuration 5: the batch-1 stack.  Every (layer, expert, tensor) has its own child seed so
# that any single expert can be regenerated without drawing the others.
# --------------------------------------------------------------------------------------------

@dataclass
class StackSpec:
    seed: int = 0
    n_layers: int = NUM_MOE_LAYERS
    d: int = D_MODEL
    f: int = D_FF
    E: int = NUM_EXPERTS
    n_codebooks: int = NUM_CODEBOOKS
    vocab_rows: int = VOCAB_ROWS
    sel_bias_var: float = 0.1
    eps: float = 1e-6
    # dense FFN layers before and after the MoE layers (the full decoder has 3 and 1); layer
    # indices below are stack positions: dense front, then the n_layers MoE layers, then dense back
    n_dense_front: int = 0
    n_dense_back: int = 0

    @property
    def total_layers(self) -> int:
        return self.n_dense_front + self.n_layers + self.n_dense_back

    def kind(self, layer: int):
        """("dense", i) for the i-th dense layer, ("moe", m) for the m-th MoE layer."""
        if layer < self.n_dense_front:
            return "dense", layer
        if layer < self.n_dense_front + self.n_layers:
            return "moe", layer - self.n_dense_front
        return "dense", layer - self.n_layers

    def E_of(self, layer: int) -> int:
        return 1 if self.kind(layer)[0] == "dense" else self.E

    def k_of(self, layer: int) -> int:
        """top-1 everywhere except top-2 in the last MoE layer."""
        kind, m = self.kind(layer)
        return 2 if kind == "moe" and m == self.n_layers - 1 else 1

    def _rng(self, *key: int) -> np.random.Generator:
        # Deterministic child stream addressed by an integer key path:
        # (0, 0) tables, (0, 1) gamma0, (1, l) layer l's router/bias/gain,
        # (2, l, e, t) expert e's tensor t of layer l, (3, 0) decode-step codes.
        return np.random.default_rng(np.random.SeedSequence(self.seed, spawn_key=tuple(key)))

    def tables(self) -> np.ndarray:
        """Embedding tables [N, V, d], N(0, 1), bf16-exact."""
        return _normal(self._rng(0, 0), (self.n_codebooks, self.vocab_rows, self.d), 1.0, True)

    def gamma0(self) -> np.ndarray:
        """Gain of the RMSNorm after the embedding sum, N(1, 0.01)."""
        return (1.0 + 0.1 * self._rng(0, 1).standard_normal(self.d, dtype=np.float32)).astype(np.float32)

    def layer_small(self, layer: int):
        """(W_r [E, d] bf16-exact, b [E] f32, gamma [d] f32) of one layer; a dense layer has no router
        (W_r and b are None)."""
        kind, m = self.kind(layer)
        if kind == "dense":
            gamma = (1.0 + 0.1 * self._rng(5, m).standard_normal(self.d, dtype=np.float32)).astype(np.float32)
            return None, None, gamma
        rng = self._rng(1, m)
        w_router = _normal(rng, (self.E, self.d), 1.0 / self.d, True)
        sel_bias = (rng.standard_normal(self.E, dtype=np.float32)
                    * np.float32(np.sqrt(self.sel_bias_var))).astype(np.float32)
        gamma = (1.0 + 0.1 * rng.standard_normal(self.d, dtype=np.float32)).astype(np.float32)
        return w_router, sel_bias, gamma

    def expert(self, layer: int, e: int):
        """(W_gate [f, d], W_up [f, d], W_down [d, f]) of one expert (the FFN of a dense layer, e = 0),
        bf16-exact."""
        kind, m = self.kind(layer)
        key = (2, m, e) if kind == "moe" else (4, m)
        wg = _normal(self._rng(*key, 0), (self.f, self.d), 1.0 / self.d, True)
        wu = _normal(self._rng(*key, 1), (self.f, self.d), 1.0 / self.d, True)
        wd = _normal(self._rng(*key, 2), (self.d, self.f), 1.0 / self.f, True)
        return wg, wu, wd

    def heads(self) -> np.ndarray:
        """Output heads [N, V, d], N(0, 1/d), bf16-exact (one bias-free linear per codebook)."""
        return _normal(self._rng(6, 0), (self.n_codebooks, self.vocab_rows, self.d), 1.0 / self.d, True)

    def gamma_out(self) -> np.ndarray:
        """Gain of the final RMSNorm before the heads, N(1, 0.01)."""
        return (1.0 + 0.1 * self._rng(6, 1).standard_normal(self.d, dtype=np.float32)).astype(np.float32)

    def codes(self, steps: int) -> np.ndarray:
        """One fresh frame of (already delay-sheared) ids per decode step: int32 [steps, N]."""
        return self._rng(3, 0).integers(0, CODEBOOK_SIZE, size=(steps, self.n_codebooks),
                                        dtype=np.int64).astype(np.int32)


# --------------------------------------------------------------------------------------------
# Bulk generation of the stack's expert weights (bf16 bit patterns), in parallel worker processes.
# --------------------------------------------------------------------------------------------

def _expert_bits_job(args):
    seed, layer, e, d, f, front, back = args
    spec = StackSpec(seed=seed, d=d, f=f, n_dense_front=front, n_dense_back=back)
    return layer, e, tuple(bf16_bits(w) for w in spec.expert(layer, e))


def stack_expert_bits(spec: StackSpec, workers: Optional[int] = None):
    """Yields (layer, expert, (W_gate, W_up, W_down) as uint16 bf16 bit arrays) for every expert of
    the stack, drawn in worker processes (spawned, so it is safe after CUDA has been initialised)."""
    import multiprocessing as mp
    import os as _os
    jobs = [(spec.seed, l, e, spec.d, spec.f, spec.n_dense_front, spec.n_dense_back)
            for l in range(spec.total_layers) for e in range(spec.E_of(l))]
    n = workers or max(1, min(16, (_os.cpu_count() or 2) - 1))
    if n == 1:
        for j in jobs:
            yield _expert_bits_job(j)
        return
    with mp.get_context("spawn").Pool(n) as pool:
        for out in pool.imap(_expert_bits_job, jobs, chunksize=2):
            yield out
