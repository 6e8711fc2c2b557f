"""zmoe_permute_noalloc through the C-ABI against zmoe_permute (the entry point with a workspace).

Some callers cannot allocate device memory at all: their framework's pool owns it, a cudaMalloc
would stall the device on a latency-critical path, or they record into a CUDA graph in a capture
mode that forbids allocation.  zmoe_permute_noalloc serves them with scratch held in a static
device array of the library.  The permutation is integer work, so its outputs must equal
zmoe_permute's bit for bit, on two calls in a row (the second call finds the array holding the
first call's contents).  This file is collected last so that a failure here leaves every other
test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_moe_decoder_b200 import zmoe_permute
from sparse_moe_decoder_b200.zmoe import ZMOE_BF16, lib
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu

OUT_KEYS = ("counts", "offsets", "perm", "inv_perm", "x_perm")


def noalloc_permute(idx: torch.Tensor, x: torch.Tensor, E: int):
    T, k = idx.shape
    d = x.shape[1]
    dev = x.device
    outs = dict(counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
                offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
                perm=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
                inv_perm=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                x_perm=torch.zeros((T * k, d), dtype=x.dtype, device=dev))
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = lib().zmoe_permute_noalloc(p(idx), p(x), ZMOE_BF16, T, d, E, k, p(outs["counts"]), p(outs["offsets"]),
                                    p(outs["perm"]), p(outs["inv_perm"]), p(outs["x_perm"]),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, outs


def case(T, E, k, seed):
    rng = np.random.default_rng(seed)
    if k == 1:
        idx = rng.integers(0, E, size=(T, 1))
    else:
        idx = np.stack([rng.permutation(E)[:2] for _ in range(T)])
    x = torch.from_numpy(rng.standard_normal((T, 256), dtype=np.float32)).to("cuda", torch.bfloat16)
    return torch.from_numpy(idx.astype(np.int32)).cuda(), x


@pytest.mark.parametrize("T,E,k", [(16384, 16, 2), (64, 16, 1), (30000, 64, 2)])
def test_noalloc_matches_workspace_entry_point_twice(T, E, k):
    require_gpu()
    for call in range(2):                         # two calls in a row share the static scratch
        idx, x = case(T, E, k, seed=100 * call + T)
        want = zmoe_permute(idx, x, E)
        st, got = noalloc_permute(idx, x, E)
        assert st == 0, lib().zmoe_last_error()
        torch.cuda.synchronize()
        for key in OUT_KEYS:
            a, b = want[key].cpu(), got[key].cpu()
            if key == "x_perm":
                a, b = a.view(torch.int16), b.view(torch.int16)
            assert torch.equal(a, b), f"call {call}: {key} differs"


def test_noalloc_rejects_sizes_beyond_its_scratch():
    require_gpu()
    T, E, k = 40000, 16, 2                        # 80000 assignments > 65536
    idx, x = case(T, E, k, seed=1)
    st, _ = noalloc_permute(idx, x, E)
    assert st == 1                                # ZMOE_ERR_INVALID_ARG, nothing launched
    assert b"65536" in lib().zmoe_last_error()
