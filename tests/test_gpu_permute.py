"""Permutation on the GPU vs the oracle: every output bit-exact, deterministic across runs."""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import round_to_bf16
from sparse_moe_decoder_b200 import zmoe_get_device_errors, zmoe_permute
from tests.gpu_util import host, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def make_idx(T, E, k, seed, skew=None):
    rng = np.random.default_rng(seed)
    if k == 1:
        if skew is not None:
            p = np.arange(1, E + 1, dtype=np.float64) ** (-skew)
            return rng.choice(E, size=(T, 1), p=p / p.sum()).astype(np.int32)
        return rng.integers(0, E, size=(T, 1)).astype(np.int32)
    return np.stack([rng.permutation(E)[:2] for _ in range(T)]).astype(np.int32)


def check(idx, x, E, dt):
    out = zmoe_permute(to_dev(idx, torch.int32), to_dev(x, dt), E)
    want = oracle.permute(idx, E, x)
    for key in ("counts", "offsets", "perm", "inv_perm"):
        assert np.array_equal(host(out[key]), want[key]), key
    rows = int(want["offsets"][-1])
    got_x = np.ascontiguousarray(host(out["x_perm"])[:rows], np.float32)
    want_x = np.ascontiguousarray(want["x_perm"][:rows], np.float32)
    assert np.array_equal(got_x.view(np.uint32), want_x.view(np.uint32))      # bit-exact copy
    return out


@pytest.mark.parametrize("T,E,k", [(1, 16, 1), (64, 16, 1), (1000, 16, 1), (512, 16, 2), (1024, 4, 1),
                                   (1025, 16, 1), (5000, 16, 2), (16384, 16, 1), (16384, 16, 2), (300, 64, 2),
                                   (0, 16, 1), (77, 1, 1)])
def test_permute_bit_exact(T, E, k):
    require_gpu()
    idx = make_idx(T, E, k, seed=T + E + k)
    x = round_to_bf16(np.random.default_rng(T).standard_normal((T, 64), dtype=np.float32))
    check(idx, x, E, torch.bfloat16)


def test_permute_skewed_and_empty_experts():
    require_gpu()
    idx = make_idx(20000, 16, 1, seed=3, skew=3.0)          # most tokens on expert 0, some experts empty
    idx[idx == 5] = 0
    x = np.random.default_rng(4).standard_normal((20000, 32), dtype=np.float32)
    check(idx, x, 16, torch.float32)


def test_permute_all_on_one_expert():
    require_gpu()
    idx = np.full((3000, 1), 7, np.int32)
    x = np.random.default_rng(5).standard_normal((3000, 16), dtype=np.float32)
    check(idx, x, 16, torch.float32)


def test_permute_deterministic():
    require_gpu()
    idx = make_idx(16384, 16, 2, seed=11)
    x = round_to_bf16(np.random.default_rng(6).standard_normal((16384, 128), dtype=np.float32))
    ref = None
    for _ in range(5):
        out = zmoe_permute(to_dev(idx, torch.int32), to_dev(x, torch.bfloat16), 16)
        cur = [host(out[k]).tobytes() for k in ("perm", "inv_perm", "x_perm")]
        if ref is None:
            ref = cur
        assert cur == ref


@pytest.mark.parametrize("T", [50, 4000])
def test_permute_bad_expert_index(T):
    """An index outside [0, E) is dropped (inv_perm = -1) and counted on the device."""
    require_gpu()
    idx = make_idx(T, 16, 1, seed=2)
    bad = [3, T // 2]
    idx[bad, 0] = [16, -1]
    x = np.random.default_rng(7).standard_normal((T, 16), dtype=np.float32)
    zmoe_get_device_errors()
    out = zmoe_permute(to_dev(idx, torch.int32), to_dev(x, torch.float32), 16)
    assert zmoe_get_device_errors() == 2
    inv = host(out["inv_perm"])
    assert (inv[bad, 0] == -1).all()
    keep = np.ones(T, bool)
    keep[bad] = False
    want = oracle.permute(idx[keep], 16, x[keep])
    assert np.array_equal(host(out["counts"]), want["counts"])
    rows = int(want["offsets"][-1])
    tokens = np.arange(T)[keep]
    assert np.array_equal(host(out["perm"])[:rows], tokens[want["perm"]])
