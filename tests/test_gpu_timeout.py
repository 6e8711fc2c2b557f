"""Failure detection on the GPU: a bounded device-side wait that runs out.

zmoe_debug_inject_timeout makes the phase-A -> phase-B hand-off of the stream-K decode layer wait for
one more finished unit than exists (a counter that nothing will raise that far), with a 5 ms limit.
The wait runs out on every CTA; each counts a timeout, stops, drains its own copies and MMAs, frees
its tensor memory and returns.  Nothing traps or faults: the host reads ZMOE_ERR_TIMEOUT from
zmoe_get_device_errors, and the next normal calls (which allocate the same tensor memory on every SM)
succeed with the result they gave before the injected failure, bit for bit.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from moe_inputs import make_config
from sparse_moe_decoder_b200 import MoELayerRunner, MoEWeights
from sparse_moe_decoder_b200.zmoe import lib
from tests.gpu_util import MARGIN_EXEMPT, assert_close, host, require_gpu, to_dev

pytestmark = pytest.mark.gpu

ZMOE_OK, ZMOE_ERR_TIMEOUT = 0, 6


def device_errors():
    c = ctypes.c_uint32(0)
    st = lib().zmoe_get_device_errors(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream), ctypes.byref(c))
    return st, int(c.value)


def test_handoff_wait_runs_out_and_the_next_call_succeeds():
    require_gpu()
    L = make_config(2)                            # T = 64: the one-launch stream-K decode layer
    W = MoEWeights.from_host(L)
    R = MoELayerRunner(L.T, L.E, L.d, L.f, L.k, torch.bfloat16)
    x = to_dev(L.x, torch.bfloat16)
    assert device_errors() == (ZMOE_OK, 0)
    good = host(R.run(x, W)).copy()
    assert device_errors() == (ZMOE_OK, 0)
    try:
        assert lib().zmoe_debug_inject_timeout(1, 5_000_000) == ZMOE_OK
        for _ in range(2):                        # twice: the second launch follows an aborted one
            R.run(x, W)
            st, n = device_errors()
            assert st == ZMOE_ERR_TIMEOUT, f"status {st}"
            assert n >= 1
    finally:
        assert lib().zmoe_debug_inject_timeout(0, 0) == ZMOE_OK
    for _ in range(3):
        again = host(R.run(x, W))
        assert device_errors() == (ZMOE_OK, 0)
        assert np.array_equal(again, good), "the layer after an aborted launch differs from before it"
    ref = oracle.moe_layer(L.x, L.w_router, L.w_gate, L.w_up, L.w_down, L.k, L.sel_bias, L.logit_bias)
    same = (host(R.idx) == ref["expert_idx"]).all(1)
    assert same[ref["margin"][:] >= MARGIN_EXEMPT].all()
    assert_close(good[same], ref["y"][same], "bf16", "layer after the timeout test")

