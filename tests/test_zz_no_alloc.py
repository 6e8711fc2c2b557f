"""zmoe_permute_noalloc through the C-ABI: against zmoe_permute (the entry point with a workspace) and
against the oracle's permutation.

Some callers cannot allocate device memory: a host framework whose pool allocator owns all of it (a
cudaMalloc behind its back can fail for lack of memory, or stall every stream while the driver maps
pages), or code on a latency-critical path that must never synchronise the device.  For them
zmoe_permute_noalloc keeps its scratch in a static device array of the library.  The permutation is
integer work and a bf16 row copy, so its outputs must equal zmoe_permute's and the oracle's bit for
bit, on two calls in a row (the second call finds the array holding the first call's contents).
Sizes up to the array's limit (T * k = 65536 assignments) are accepted, one past it is rejected.
This file is collected last so that a failure here leaves every other test already run.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from sparse_moe_decoder_b200 import zmoe_permute
from sparse_moe_decoder_b200.zmoe import ZMOE_BF16, lib
from tests.gpu_util import require_gpu

pytestmark = pytest.mark.gpu

OUT_KEYS = ("counts", "offsets", "perm", "inv_perm", "x_perm")
LIMIT = 65536                                     # assignments the static scratch holds


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
        idx = np.argsort(rng.random((T, E)), axis=1)[:, :2]      # two distinct experts per token
    x = rng.standard_normal((T, 256), dtype=np.float32)
    return idx.astype(np.int32), x


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy()


@pytest.mark.parametrize("T,E,k", [(16384, 16, 2), (64, 16, 1), (30000, 64, 2), (32768, 16, 2), (65536, 4, 1)])
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(T, E, k):
    require_gpu()
    for call in range(2):                         # two calls in a row share the static scratch
        idx_h, x_h = case(T, E, k, seed=100 * call + T)
        idx = torch.from_numpy(idx_h).cuda()
        x = torch.from_numpy(x_h).to("cuda", torch.bfloat16)
        want = zmoe_permute(idx, x, E)
        st, got = noalloc_permute(idx, x, E)
        assert st == 0, lib().zmoe_last_error()
        torch.cuda.synchronize()
        for key in OUT_KEYS:
            a, b = want[key], got[key]
            if key == "x_perm":
                assert np.array_equal(bf16_bits(a), bf16_bits(b)), f"call {call}: {key} differs from zmoe_permute"
            else:
                assert torch.equal(a.cpu(), b.cpu()), f"call {call}: {key} differs from zmoe_permute"
        ref = oracle.permute(idx_h, E, x.float().cpu().numpy())
        for key in ("counts", "offsets", "perm", "inv_perm"):
            assert np.array_equal(got[key].cpu().numpy(), ref[key]), f"call {call}: {key} differs from the oracle"
        x_ref = torch.from_numpy(np.ascontiguousarray(ref["x_perm"], np.float32)).to(torch.bfloat16)
        assert np.array_equal(bf16_bits(got["x_perm"]), x_ref.view(torch.int16).numpy()), \
            f"call {call}: x_perm differs from the oracle"


@pytest.mark.parametrize("T,k", [(32769, 2), (LIMIT + 1, 1)])
def test_noalloc_rejects_sizes_beyond_its_scratch(T, k):
    require_gpu()
    E = 16
    assert T * k == LIMIT + 1 or T * k == LIMIT + 2
    idx_h, x_h = case(T, E, k, seed=1)
    idx = torch.from_numpy(idx_h).cuda()
    x = torch.from_numpy(x_h).to("cuda", torch.bfloat16)
    st, out = noalloc_permute(idx, x, E)
    assert st == 1                                # ZMOE_ERR_INVALID_ARG, nothing launched
    assert b"65536" in lib().zmoe_last_error()
    torch.cuda.synchronize()
    assert int(out["counts"][0]) == -7            # outputs untouched
