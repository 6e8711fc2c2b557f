"""zmoe_moe_layer (one call per MoE layer; one cooperative launch at decode sizes) vs the oracle.

The fused decode launch forms, in one kernel: the optional pre-norm, the router, the dispatch
permutation, the SwiGLU and the combine.  Each case is checked on every token:
  * expert ids bit-exact except where the fp64 selection margin is below 1e-4 (reported);
  * gates within 1e-4, on the tokens whose ids agree;
  * the layer's MoE output y - h held to the bf16 bar, max |err| <= 2e-2 x RMS, against the
    oracle run on the GPU's own routed input x (the pre-norm output is bf16: rounding it is part
    of the method, and the oracle consumes the same bf16 values);
  * with the pre-norm, x itself against the fp64 RMSNorm, and the result in place (y aliasing h).
Shapes span one and several 16-row token blocks per expert, top-1 and top-2, E = 1, an empty
expert, batch 1, the tiny-batch launch (T * k <= 4) and its boundary, and the full decode-step size.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import make_moe_layer
from sparse_moe_decoder_b200 import MoELayerRunner, MoEWeights, zmoe_get_device_errors
from tests.gpu_util import MARGIN_EXEMPT, assert_close, host, rel_err, require_gpu, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-6

# (T, d, f, E, k, selection-bias variance): all on the fused path (bf16, T*k < 64 E, T*k <= 1024)
CASES = [
    (1, 256, 256, 16, 1, 0.1),
    (1, 256, 512, 16, 2, 0.1),
    (3, 512, 256, 4, 2, 0.0),
    (17, 256, 256, 16, 1, 0.1),
    (40, 256, 256, 1, 1, 0.0),
    (64, 256, 512, 16, 2, 0.1),
    (200, 256, 256, 8, 2, 0.5),
    (600, 256, 256, 16, 1, 0.5),
]


def check_layer(L, h, y, idx, gates, x_routed, what):
    """y = h + MoE(x_routed) against the oracle on the GPU's routed input."""
    ref = oracle.moe_layer(x_routed, L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)
    ok = ref["margin"] >= MARGIN_EXEMPT
    assert np.array_equal(idx[ok], ref["expert_idx"][ok]), f"{what}: routing differs on a token with margin >= 1e-4"
    same = (idx == ref["expert_idx"]).all(1)
    assert np.max(np.abs(gates[same] - ref["gates"][same]), initial=0.0) <= 1e-4, f"{what}: gates"
    moe = y - (h if h is not None else 0.0)
    r = assert_close(moe[same], ref["y"][same], "bf16", f"{what}: y - h")
    return r, int((~ok).sum())


def run_fused(L, h_host=None, gamma=None, in_place=False):
    dt = torch.bfloat16
    W = MoEWeights.from_host(L)
    T, d = L.x.shape
    R = MoELayerRunner(T, L.E, d, L.f, L.k, dt)
    h = to_dev(h_host, torch.float32) if h_host is not None else None
    x_norm = torch.empty((T, d), dtype=dt, device="cuda") if gamma is not None else None
    out = h if in_place else None
    y = R.run(None if gamma is not None else to_dev(L.x, dt), W, residual=h, out=out,
              gamma=to_dev(gamma, torch.float32) if gamma is not None else None, eps=EPS, x_norm=x_norm)
    torch.cuda.synchronize()
    assert zmoe_get_device_errors() == 0
    return R, host(y).astype(np.float64), (host(x_norm).astype(np.float64) if x_norm is not None else None)


@pytest.mark.parametrize("T,d,f,E,k,sv", CASES)
def test_fused_layer_with_residual(T, d, f, E, k, sv):
    require_gpu()
    L = make_moe_layer(T, d, f, E, k, seed=T + 7 * E + k, sel_bias_var=sv)
    h = np.random.default_rng(T).standard_normal((T, d)).astype(np.float32)
    R, y, _ = run_fused(L, h_host=h)
    r, ex = check_layer(L, h.astype(np.float64), y, host(R.idx), host(R.gates), L.x.astype(np.float64),
                        f"T={T} d={d} f={f} E={E} k={k}")
    print(f"T={T} d={d} f={f} E={E} k={k}: y-h max err {r:.2e} x RMS, {ex} low-margin tokens")


@pytest.mark.parametrize("T,d,f,E,k,sv", CASES[:6])
def test_fused_layer_prenorm_in_place(T, d, f, E, k, sv):
    """h <- h + MoE(RMSNorm(h) * gamma), y written over h (the decode stack's layer)."""
    require_gpu()
    L = make_moe_layer(T, d, f, E, k, seed=100 + T + E, sel_bias_var=sv, with_gamma=True, draw_x=False)
    h = (3.0 * np.random.default_rng(T + 1).standard_normal((T, d))).astype(np.float32)
    R, y, xn = run_fused(L, h_host=h, gamma=L.gamma, in_place=True)
    assert_close(xn, oracle.rmsnorm(h.astype(np.float64), L.gamma.astype(np.float64), EPS), "bf16",
                 "pre-norm output")
    r, ex = check_layer(L, h.astype(np.float64), y, host(R.idx), host(R.gates), xn, f"prenorm T={T} E={E} k={k}")
    print(f"prenorm T={T} E={E} k={k}: y-h max err {r:.2e} x RMS, {ex} low-margin tokens")


def test_fused_layer_empty_experts_and_no_residual():
    """Every token forced onto expert 2 of 8 (selection bias): seven experts get no rows."""
    require_gpu()
    L = make_moe_layer(33, 256, 256, 8, 1, seed=5)
    L.sel_bias = np.full(8, -100.0, np.float32)
    L.sel_bias[2] = 100.0
    R, y, _ = run_fused(L)
    assert (host(R.idx) == 2).all()
    check_layer(L, None, y, host(R.idx), host(R.gates), L.x.astype(np.float64), "one expert")


@pytest.mark.parametrize("k", [1, 2])
def test_fused_layer_full_size(k):
    """The decode-step size: T = 64, d_model 2048, d_ff 3072, 16 experts."""
    require_gpu()
    L = make_moe_layer(64, 2048, 3072, 16, k, seed=11 + k, sel_bias_var=0.1)
    h = np.random.default_rng(k).standard_normal((64, 2048)).astype(np.float32)
    R, y, _ = run_fused(L, h_host=h)
    r, ex = check_layer(L, h.astype(np.float64), y, host(R.idx), host(R.gates), L.x.astype(np.float64),
                        f"full size k={k}")
    print(f"full size k={k}: y-h max err {r:.2e} x RMS, {ex} low-margin tokens")


@pytest.mark.parametrize("T,k", [(1, 1), (64, 1), (64, 2), (300, 2)])
def test_fused_matches_separate_calls(T, k):
    """The one-launch layer and the four separate entry points agree (same FFN arithmetic; the
    router's fp32 summation order differs, so ids may differ only on near-ties)."""
    require_gpu()
    L = make_moe_layer(T, 512, 512, 16, k, seed=T + k, sel_bias_var=0.1)
    dt = torch.bfloat16
    W = MoEWeights.from_host(L)
    x = to_dev(L.x, dt)
    h = to_dev(np.random.default_rng(3).standard_normal((T, 512)).astype(np.float32), torch.float32)
    R1 = MoELayerRunner(T, 16, 512, 512, k, dt)
    R2 = MoELayerRunner(T, 16, 512, 512, k, dt)
    y1 = host(R1.run(x, W, residual=h)).astype(np.float64)
    y2 = host(R2.run_steps(x, W, residual=h)).astype(np.float64)
    same = (host(R1.idx) == host(R2.idx)).all(1)
    assert same.mean() >= 0.98
    assert rel_err(y1[same], y2[same]) <= 1e-4


def test_fused_repeatable_bitwise():
    require_gpu()
    L = make_moe_layer(64, 512, 512, 16, 2, seed=9, sel_bias_var=0.1)
    dt = torch.bfloat16
    W = MoEWeights.from_host(L)
    R = MoELayerRunner(64, 16, 512, 512, 2, dt)
    x = to_dev(L.x, dt)
    first = host(R.run(x, W)).copy()
    for _ in range(3):
        assert np.array_equal(host(R.run(x, W)), first)


@pytest.mark.parametrize("T,k", [(2, 2), (4, 1), (2, 1), (5, 1)])
def test_tiny_batch_layer(T, k):
    """A few tokens (T * k <= 4 runs the tiny-batch launch, T = 5 the stream-K one): the decode
    stack's pre-norm layer in place, at the model's dimensions, against the oracle."""
    require_gpu()
    L = make_moe_layer(T, 2048, 3072, 16, k, seed=70 + T + k, sel_bias_var=0.1, with_gamma=True, draw_x=False)
    h = (2.0 * np.random.default_rng(T).standard_normal((T, 2048))).astype(np.float32)
    R, y, xn = run_fused(L, h_host=h, gamma=L.gamma, in_place=True)
    assert_close(xn, oracle.rmsnorm(h.astype(np.float64), L.gamma.astype(np.float64), EPS), "bf16", "pre-norm output")
    r, ex = check_layer(L, h.astype(np.float64), y, host(R.idx), host(R.gates), xn, f"tiny T={T} k={k}")
    print(f"tiny T={T} k={k}: y-h max err {r:.2e} x RMS, {ex} low-margin tokens")


@pytest.mark.parametrize("T", [1, 40, 300])
def test_dense_layer_without_router(T):
    """E = 1 and no router: the decoder's dense FFN layers, h <- h + SwiGLU(RMSNorm(h) * gamma)
    (fused below 64 tokens, the separate entry points above)."""
    require_gpu()
    L = make_moe_layer(T, 512, 512, 1, 1, seed=T, with_gamma=True, draw_x=False)
    h = np.random.default_rng(T).standard_normal((T, 512)).astype(np.float32)
    dt = torch.bfloat16
    W = MoEWeights.from_host(L)
    W.w_router = None
    W.sel_bias = None
    R = MoELayerRunner(T, 1, 512, 512, 1, dt)
    hd = to_dev(h, torch.float32)
    xn = torch.empty((T, 512), dtype=dt, device="cuda")
    y = host(R.run(None, W, residual=hd, out=hd, gamma=to_dev(L.gamma, torch.float32), eps=EPS,
                   x_norm=xn)).astype(np.float64)
    torch.cuda.synchronize()
    assert zmoe_get_device_errors() == 0
    assert (host(R.idx) == 0).all() and (host(R.gates) == 1.0).all()
    x = host(xn).astype(np.float64)
    assert_close(x, oracle.rmsnorm(h.astype(np.float64), L.gamma.astype(np.float64), EPS), "bf16", "pre-norm")
    want = oracle.swiglu_ffn(x, L.w_gate[0], L.w_up[0], L.w_down[0])
    assert_close(y - h, want, "bf16", f"dense layer T={T}")
