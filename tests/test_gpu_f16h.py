"""The prefill path with h carried in f16 and the prepared f16 down weights, through the C-ABI.

zmoe_prepare_w_down_f16 is checked against its definition: w_down = w_down_f16 * down_scale exactly for
every weight within 2^28 of its expert's largest (bit-exact as doubles), with a power-of-two scale per
expert.  The grouped SwiGLU and the whole layer are checked against the fp64 oracle on every row and
token: y_perm and y within the bf16 bar (2e-2 x RMS), routing ids bit-exact outside the margin exemption.
h is checked against f16's own rounding bound: |h_gpu - h| <= 2^-11 |h| (half an f16 ulp, relative to each
element: h has tails ~30x its RMS) plus 1e-3 x RMS(h) for the fp32 accumulation of bf16 products over
K = d (~1.5e-4 x RMS measured).  An h beyond f16's range is counted as a device error.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import make_config, make_moe_layer
from sparse_moe_decoder_b200 import (MoELayerRunner, MoEWeights, zmoe_get_device_errors, zmoe_grouped_swiglu_f16h,
                                     zmoe_prepare_w_down_f16)
from tests.gpu_util import MARGIN_EXEMPT, assert_close, host, require_gpu, to_dev

pytestmark = pytest.mark.gpu

H16_TOL = 1e-3


def check_h16(h, h_ref):
    """max(|h - h_ref| - 2^-11 |h_ref|) <= 1e-3 x RMS(h_ref); returns that excess / RMS."""
    h_ref = np.asarray(h_ref, np.float64)
    rms = float(np.sqrt(np.mean(h_ref * h_ref)))
    excess = float(np.max(np.abs(np.asarray(h, np.float64) - h_ref) - 2.0 ** -11 * np.abs(h_ref))) / rms
    assert excess <= H16_TOL, f"h (f16): error beyond half an f16 ulp = {excess:.3e} x RMS"
    return excess


def _offsets(counts):
    return np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)


def run_f16h(L, x_perm, offsets):
    W = MoEWeights.from_host(L).prepare_f16()
    h, y = zmoe_grouped_swiglu_f16h(to_dev(x_perm, torch.bfloat16), to_dev(offsets, torch.int32), W.w_gate, W.w_up,
                                    W.w_down_f16, W.down_scale)
    return host(h.float()), host(y)


def test_prepare_w_down_f16_is_exact():
    require_gpu()
    rng = np.random.default_rng(7)
    E, d, f = 5, 256, 512
    w = rng.standard_normal((E, d, f), dtype=np.float32) / np.sqrt(f)
    w[1] *= 1e-6                                      # a tiny expert
    w[2] *= 3e4                                       # a huge one (beyond f16 range before scaling)
    w[3] = 0.0                                        # an all-zero expert
    w[4, 0, :8] = [1e-20, -1e-20, 0.5, -0.5, 2.0 ** -30, 0.0, 1.0, -1.0]
    wb = torch.from_numpy(w).to(torch.bfloat16).cuda()
    w16, sc = zmoe_prepare_w_down_f16(wb)
    torch.cuda.synchronize()
    want = wb.double().cpu().numpy()
    got = w16.double().cpu().numpy() * sc.double().cpu().numpy()[:, None, None]
    s = sc.cpu().numpy().astype(np.float64)
    assert np.all(np.log2(s) == np.round(np.log2(s))), "scales must be powers of two"
    for e in range(E):
        amax = np.abs(want[e]).max()
        if amax == 0:
            assert s[e] == 1.0 and np.all(got[e] == 0)
            continue
        scaled_max = amax / s[e]
        assert 2.0 ** 14 <= scaled_max < 2.0 ** 15, f"expert {e}: largest |w| scaled to {scaled_max}"
        e_max = np.floor(np.log2(amax))
        big = np.abs(want[e]) >= 2.0 ** (e_max - 28)
        assert np.array_equal(got[e][big], want[e][big]), f"expert {e}: not exact"
        assert np.all(np.abs(got[e][~big] - want[e][~big]) <= 2.0 ** (e_max - 39))


@pytest.mark.parametrize("counts", [
    [0, 5, 0, 1, 9, 0, 0, 33, 2, 0, 0, 0, 8, 0, 0, 1],       # empty experts, tiny segments
    [300, 0, 129, 700, 64, 1, 255, 257, 0, 0, 0, 0, 0, 0, 0, 40],   # 256-row tile edges +-1
])
def test_f16h_ragged_rows(counts):
    require_gpu()
    M = int(sum(counts))
    L = make_moe_layer(M, 2048, 3072, 16, 1, "bf16", seed=M + 11)
    off = _offsets(counts)
    h, y = run_f16h(L, L.x, off)
    y_ref, h_ref = oracle.grouped_swiglu(L.x, off, L.w_gate, L.w_up, L.w_down)
    assert_close(y, y_ref, "bf16", "ragged y_perm (f16 h)")
    check_h16(h, h_ref)


@pytest.mark.parametrize("E,d,f,counts", [
    (1, 256, 256, [64]),
    (4, 2048, 2048, [2500, 1800, 3100, 792]),        # ~540 gate/up tiles over 74 CTA pairs
    (16, 512, 512, [0] * 15 + [1500]),
])
def test_f16h_tensor_core_shapes(E, d, f, counts):
    require_gpu()
    M = int(sum(counts))
    L = make_moe_layer(M, d, f, E, 1, "bf16", seed=M + d + 1)
    off = _offsets(counts)
    h, y = run_f16h(L, L.x, off)
    y_ref, h_ref = oracle.grouped_swiglu(L.x, off, L.w_gate, L.w_up, L.w_down)
    r = assert_close(y, y_ref, "bf16", "f16h y_perm")
    check_h16(h, h_ref)
    print(f"f16h E={E} d={d} f={f}: y_perm max err {r:.2e} x RMS")


def test_f16h_single_expert_equals_dense_ffn():
    require_gpu()
    L = make_moe_layer(300, 1024, 512, 1, 1, "bf16", seed=9)
    off = np.array([0, 300], np.int32)
    _, y = run_f16h(L, L.x, off)
    assert_close(y, oracle.swiglu_ffn(L.x, L.w_gate[0], L.w_up[0], L.w_down[0]), "bf16", "dense FFN (f16 h)")


@pytest.mark.parametrize("cfg", [3, 4])
def test_f16h_prefill_every_row(cfg):
    require_gpu()
    L = make_config(cfg)
    sel, gates, margin, _ = oracle.route(L.x, L.w_router, L.k, L.sel_bias, L.logit_bias)
    p = oracle.permute(sel, L.E, L.x)
    h, y = run_f16h(L, p["x_perm"], p["offsets"])
    y_ref, h_ref = oracle.grouped_swiglu(p["x_perm"], p["offsets"], L.w_gate, L.w_up, L.w_down)
    r = assert_close(y, y_ref, "bf16", f"config {cfg} y_perm (f16 h, every row)")
    rh = check_h16(h, h_ref)
    print(f"config {cfg}: f16h y_perm max err {r:.2e} x RMS, h excess over half an ulp {rh:.2e} x RMS over {y.shape[0]} rows")


@pytest.mark.parametrize("cfg", [3, 4])
@pytest.mark.parametrize("steps", [False, True], ids=["one_call", "separate_calls"])
def test_layer_f16h_every_token(cfg, steps):
    require_gpu()
    L = make_config(cfg)
    W = MoEWeights.from_host(L).prepare_f16()
    R = MoELayerRunner(L.T, L.E, L.d, L.f, L.k, torch.bfloat16)
    x = to_dev(L.x, torch.bfloat16)
    y = host(R.run_steps_f16h(x, W) if steps else R.run_f16h(x, W))
    ref = oracle.moe_layer(L.x, L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)
    idx = host(R.idx)
    ok = ref["margin"] >= MARGIN_EXEMPT
    assert np.array_equal(idx[ok], ref["expert_idx"][ok])
    same = (idx == ref["expert_idx"]).all(1)
    r = assert_close(y[same], ref["y"][same], "bf16", f"config {cfg} y (f16 h)")
    assert zmoe_get_device_errors() == 0
    print(f"config {cfg}: f16h layer y max err {r:.2e} x RMS over {int(same.sum())} tokens")


def test_f16h_range_overflow_is_counted():
    """Inputs 300x larger push |h| past 65504: counted on the device, no fault."""
    require_gpu()
    L = make_moe_layer(512, 256, 256, 2, 1, "bf16", seed=3)
    x = L.x * 300.0
    off = np.array([0, 300, 512], np.int32)
    assert zmoe_get_device_errors() == 0
    run_f16h(L, x, off)
    assert zmoe_get_device_errors() >= 1
