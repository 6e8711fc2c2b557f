"""The codebook output heads + greedy next frame on the GPU vs the oracle.

The input x (the final RMSNorm of h, rounded to bf16) is held to the bf16 bar against the fp64 RMSNorm;
the logits, formed from the GPU's own x, to the fp32 bar (max |err| <= 1e-4 x RMS); the ids bit-exact
except where the oracle's top-two logit margin is below 1e-4 (counted).  Full size: 9 heads of
1025 x 2048, T = 1 (the decode step), 8 (one pass) and 13 (two passes over the weights).
"""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import StackSpec
from sparse_moe_decoder_b200 import zmoe_get_device_errors, zmoe_output_heads
from tests.gpu_util import MARGIN_EXEMPT, TOL, assert_close, host, rel_err, require_gpu, to_dev

pytestmark = pytest.mark.gpu

EPS = 1e-6


@pytest.fixture(scope="module")
def heads():
    require_gpu()
    spec = StackSpec()
    return spec, spec.heads(), to_dev(spec.heads(), torch.bfloat16), spec.gamma_out()


@pytest.mark.parametrize("T", [1, 8, 13])
def test_heads_full_size(heads, T):
    spec, W, Wd, g = heads
    h = (2.0 * np.random.default_rng(T).standard_normal((T, spec.d))).astype(np.float32)
    out = zmoe_output_heads(to_dev(h, torch.float32), Wd, to_dev(g, torch.float32), EPS, want_logits=True,
                            want_x=True)
    torch.cuda.synchronize()
    assert zmoe_get_device_errors() == 0
    x = host(out["x"]).astype(np.float64)
    assert_close(x, oracle.rmsnorm(h.astype(np.float64), g, EPS), "bf16", "final norm")
    ref = oracle.output_heads(h, W, g, EPS, x_rounded=x)
    r = rel_err(host(out["logits"]), ref["logits"])
    assert r <= TOL["f32"], f"logits {r:.2e} x RMS"
    ok = ref["margin"] >= MARGIN_EXEMPT
    ids = host(out["ids"])
    assert np.array_equal(ids[ok], ref["ids"][ok])
    print(f"heads T={T}: logits max err {r:.2e} x RMS, {int((~ok).sum())} low-margin (token, codebook) exempt")


def test_heads_exact_tie_across_ctas_lower_id():
    """Rows 1 and 3 of codebook 0 give the same (largest) logit: the lower id wins, whichever of the
    CTAs holding them finishes first; codebook 1 has a unique maximum."""
    require_gpu()
    N, V, d = 2, 5, 16
    W = np.zeros((N, V, d), np.float32)
    W[0, 1] = W[0, 3] = 1.0
    W[0, 0] = 0.5
    W[0, 4] = -1.0
    W[1, 2] = 2.0
    W[1, 0] = 1.0
    h = np.ones((3, d), np.float32)
    out = zmoe_output_heads(to_dev(h, torch.float32), to_dev(W, torch.bfloat16), want_logits=True)
    ids = host(out["ids"])
    assert ids.tolist() == [[1, 2]] * 3
    assert np.array_equal(host(out["logits"]), oracle.head_logits(h, W))


def test_heads_f32_weights():
    require_gpu()
    rng = np.random.default_rng(5)
    N, V, d, T = 3, 77, 96, 5
    W = rng.standard_normal((N, V, d)).astype(np.float32)
    h = rng.standard_normal((T, d)).astype(np.float32)
    g = (1 + 0.1 * rng.standard_normal(d)).astype(np.float32)
    out = zmoe_output_heads(to_dev(h, torch.float32), to_dev(W, torch.float32), to_dev(g, torch.float32), EPS,
                            want_logits=True, want_x=True)
    x = host(out["x"]).astype(np.float64)
    assert_close(x, oracle.rmsnorm(h.astype(np.float64), g, EPS), "f32", "final norm (f32)")
    ref = oracle.output_heads(h, W, g, EPS, x_rounded=x)
    assert rel_err(host(out["logits"]), ref["logits"]) <= TOL["f32"]
    ok = ref["margin"] >= MARGIN_EXEMPT
    assert np.array_equal(host(out["ids"])[ok], ref["ids"][ok])
