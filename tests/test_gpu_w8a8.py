"""The W8A8 fp8 prefill layer (zmoe_moe_layer_w8a8) through the C-ABI vs the oracle's W8A8 layer.

The oracle quantizes the same way (per-token dynamic scales for the token rows and the f16-held hidden
rows, E4M3 codes by round to nearest even), taking the scale and the quotient in fp32 like the kernel, so
the token-row codes agree exactly; the hidden rows' codes can differ where the kernel's fp32 h and the
oracle's fp64 h round to different E4M3 neighbours (rare; each moves one element by one E4M3 step).  The bar
is the bf16 one: max |y_gpu - y_oracle| <= 2e-2 x RMS on every token whose routing agrees; ids bit-exact
outside the 1e-4 margin exemption.  The effect of the quantization itself (against the bf16 layer) is
printed, not asserted.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import make_config, make_moe_layer, quantize_e4m3_rows
from sparse_moe_decoder_b200 import zmoe_get_device_errors, zmoe_moe_layer_w8a8
from tests.gpu_util import MARGIN_EXEMPT, assert_close, host, rel_err, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def run(L, residual=None):
    Q = [quantize_e4m3_rows(w) for w in (L.w_gate, L.w_up, L.w_down)]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    idx = torch.empty((L.T, L.k), dtype=torch.int32, device="cuda")
    y = zmoe_moe_layer_w8a8(to_dev(L.w_router, torch.bfloat16), dev(Q[0][0]), dev(Q[0][1]), dev(Q[1][0]),
                            dev(Q[1][1]), dev(Q[2][0]), dev(Q[2][1]), L.k, x=to_dev(L.x, torch.bfloat16),
                            h=None if residual is None else to_dev(residual, torch.float32),
                            sel_bias=None if L.sel_bias is None else dev(L.sel_bias),
                            logit_bias=None if L.logit_bias is None else dev(L.logit_bias),
                            outs=dict(expert_idx=idx))
    ref = oracle.moe_layer_w8a8(L.x, L.w_router, Q[0][0], Q[0][1], Q[1][0], Q[1][1], Q[2][0], Q[2][1], L.k,
                                sel_bias=L.sel_bias, logit_bias=L.logit_bias, residual=residual)
    return host(y), host(idx), ref


def check(L, what, residual=None):
    y, idx, ref = run(L, residual)
    ok = ref["margin"] >= MARGIN_EXEMPT
    assert np.array_equal(idx[ok], ref["expert_idx"][ok]), f"{what}: routing differs"
    same = (idx == ref["expert_idx"]).all(1)
    r = assert_close(y[same], ref["y"][same], "bf16", f"{what} y (W8A8)")
    assert zmoe_get_device_errors() == 0
    return y, ref, r, same


@pytest.mark.parametrize("cfg", [3, 4])
def test_w8a8_prefill_every_token(cfg):
    require_gpu()
    L = make_config(cfg)
    y, ref, r, same = check(L, f"config {cfg}")
    bf = oracle.moe_layer(L.x, L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)["y"]
    print(f"config {cfg}: W8A8 y max err {r:.2e} x RMS vs the W8A8 oracle over {int(same.sum())} tokens; "
          f"quantization moves the layer by {rel_err(ref['y'], bf):.3f} x RMS vs bf16")


@pytest.mark.parametrize("T,E,k", [(300, 4, 1), (1500, 16, 2), (64, 1, 1)])
def test_w8a8_small_shapes_with_residual(T, E, k):
    require_gpu()
    L = make_moe_layer(T, 256, 512, E, k, "bf16", seed=T + E)
    res = np.random.default_rng(T).standard_normal((T, 256)).astype(np.float32)
    check(L, f"T={T} E={E} k={k}", residual=res)
