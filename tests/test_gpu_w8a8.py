"""The W8A8 fp8 prefill layer (zmoe_moe_layer_w8a8) through the C-ABI against the oracle, step by step.

Quantization turns floating point into integer decisions (E4M3 codes), so each decision is compared where
both sides take it on identical inputs and in the same precision, and the floating-point steps between
them are compared within their own rounding (teacher forcing, as for the decode stack):
  * routing: ids bit-exact outside the 1e-4 margin exemption; the permutation of the GPU's ids bit-exact;
  * token rows: the oracle's per-token quantization of the GPU-permuted rows gives the GPU's codes and
    scales exactly (the scale and quotient in fp32 on both sides);
  * h: the oracle's fp64 hidden rows from those codes are within half an f16 ulp (+1e-3 x RMS for the fp32
    accumulation) of the GPU's f16 h;
  * hidden rows: the oracle's quantization of the GPU's own f16 h gives the GPU's codes and scales exactly;
  * y_perm: the oracle's down projection of the GPU's hidden codes is within 1e-3 x RMS (fp32 accumulation
    only), and y within the bf16 bar (2e-2 x RMS).
Free-running (the oracle quantizing its own fp64 h), a hidden value that lies within the fp32 error of an
E4M3 rounding midpoint may round to the other neighbour on each side; such flips are counted and the
free-running error printed, not asserted.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import make_config, make_moe_layer, quantize_e4m3_rows
from sparse_moe_decoder_b200 import zmoe_get_device_errors, zmoe_moe_layer_w8a8
from sparse_moe_decoder_b200.zmoe import lib, w8a8_intermediates
from tests.gpu_util import MARGIN_EXEMPT, assert_close, host, rel_err, require_gpu, to_dev

pytestmark = pytest.mark.gpu

H16_TOL = 1e-3


def run(L, residual=None):
    Q = [quantize_e4m3_rows(w) for w in (L.w_gate, L.w_up, L.w_down)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    idx = torch.empty((L.T, L.k), dtype=torch.int32, device="cuda")
    gates = torch.empty((L.T, L.k), dtype=torch.float32, device="cuda")
    ws = torch.empty(int(lib().zmoe_moe_layer_w8a8_workspace_size(L.T, L.d, L.f, L.E, L.k)), dtype=torch.uint8,
                     device="cuda")
    y = zmoe_moe_layer_w8a8(to_dev(L.w_router, torch.bfloat16), dev(Q[0][0]), dev(Q[0][1]), dev(Q[1][0]),
                            dev(Q[1][1]), dev(Q[2][0]), dev(Q[2][1]), L.k, x=to_dev(L.x, torch.bfloat16),
                            h=None if residual is None else to_dev(residual, torch.float32),
                            sel_bias=None if L.sel_bias is None else dev(L.sel_bias),
                            logit_bias=None if L.logit_bias is None else dev(L.logit_bias),
                            outs=dict(expert_idx=idx, gates=gates), workspace=ws)
    torch.cuda.synchronize()
    mid = {k_: host(v.float()) if v.dtype == torch.float16 else v.cpu().numpy()
           for k_, v in w8a8_intermediates(ws, L.T, L.d, L.f, L.E, L.k).items()}
    return host(y), host(idx), host(gates), mid, Q


def check_layer(L, what, residual=None):
    y, idx, gates, mid, Q = run(L, residual)
    assert zmoe_get_device_errors() == 0
    sel, g_ref, margin, _ = oracle.route(L.x, L.w_router, L.k, L.sel_bias, L.logit_bias)
    ok = margin >= MARGIN_EXEMPT
    assert np.array_equal(idx[ok], sel[ok]), f"{what}: routing differs on a token with margin >= 1e-4"
    # the permutation of the GPU's own ids
    p = oracle.permute(idx, L.E, L.x)
    for key in ("counts", "offsets", "perm", "inv_perm"):
        assert np.array_equal(mid[key], p[key]), f"{what}: {key}"
    off = p["offsets"]
    # token rows: codes and scales exactly
    qx, sx = oracle.quantize_rows_dynamic(p["x_perm"])
    assert np.array_equal(mid["sx"], sx), f"{what}: token scales differ"
    assert np.array_equal(oracle.e4m3_decode(mid["xq"]), oracle.e4m3_decode(qx)), f"{what}: token codes differ"
    # h from those codes, in fp64
    xq = oracle.e4m3_decode(qx) * sx[:, None].astype(np.float64)
    h_ref = np.zeros((xq.shape[0], L.f))
    for e in range(L.E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            gg = xq[a:b] @ oracle.dequantize_rows(Q[0][0][e], Q[0][1][e]).T
            uu = xq[a:b] @ oracle.dequantize_rows(Q[1][0][e], Q[1][1][e]).T
            h_ref[a:b] = oracle.silu(gg) * uu
    rms = float(np.sqrt(np.mean(h_ref * h_ref)))
    excess = float(np.max(np.abs(mid["h16"] - h_ref) - 2.0 ** -11 * np.abs(h_ref))) / rms
    assert excess <= H16_TOL, f"{what}: h beyond half an f16 ulp by {excess:.2e} x RMS"
    # hidden rows: the oracle's quantization of the GPU's own f16 h gives the GPU's codes and scales
    qh, sh = oracle.quantize_rows_dynamic(mid["h16"].astype(np.float32))
    assert np.array_equal(mid["sh"], sh), f"{what}: hidden scales differ"
    assert np.array_equal(oracle.e4m3_decode(mid["hq"]), oracle.e4m3_decode(qh)), f"{what}: hidden codes differ"
    # the down projection of those codes, and the combine
    hq = oracle.e4m3_decode(qh) * sh[:, None].astype(np.float64)
    yp_ref = np.zeros((hq.shape[0], L.d))
    for e in range(L.E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            yp_ref[a:b] = hq[a:b] @ oracle.dequantize_rows(Q[2][0][e], Q[2][1][e]).T
    r_yp = rel_err(mid["y_perm"], yp_ref)
    assert r_yp <= 1e-3, f"{what}: y_perm {r_yp:.2e} x RMS"
    y_ref = oracle.combine(yp_ref, p["inv_perm"], gates.astype(np.float64), residual)
    assert_close(y, y_ref, "bf16", f"{what} y (teacher-forced)")
    # free-running: report only
    free = oracle.moe_layer_w8a8(L.x, L.w_router, Q[0][0], Q[0][1], Q[1][0], Q[1][1], Q[2][0], Q[2][1], L.k,
                                 sel_bias=L.sel_bias, logit_bias=L.logit_bias, residual=residual)
    same = (idx == free["expert_idx"]).all(1)
    flips = int(np.sum(oracle.e4m3_decode(free["qh"]) != oracle.e4m3_decode(mid["hq"]))) \
        if np.array_equal(free["perm"], p["perm"]) else -1
    print(f"{what}: y_perm {r_yp:.2e} x RMS (teacher-forced); free-running y max err "
          f"{rel_err(y[same], free['y'][same]):.2e} x RMS with {flips} hidden-code flips of {mid['hq'].size}")
    return y, free


@pytest.mark.parametrize("cfg", [3, 4])
def test_w8a8_prefill_every_token(cfg):
    require_gpu()
    L = make_config(cfg)
    y, free = check_layer(L, f"config {cfg}")
    bf = oracle.moe_layer(L.x, L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)["y"]
    print(f"config {cfg}: W8A8 quantization moves the layer by {rel_err(free['y'], bf):.3f} x RMS vs bf16")


@pytest.mark.parametrize("T,E,k", [(300, 4, 1), (1500, 16, 2), (64, 1, 1)])
def test_w8a8_small_shapes_with_residual(T, E, k):
    require_gpu()
    L = make_moe_layer(T, 256, 512, E, k, "bf16", seed=T + E)
    res = np.random.default_rng(T).standard_normal((T, 256)).astype(np.float32)
    check_layer(L, f"T={T} E={E} k={k}", residual=res)
