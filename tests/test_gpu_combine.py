"""Combine on the GPU vs the oracle (fp32 results; deterministic gather)."""
import numpy as np
import pytest
import torch

import oracle
from sparse_moe_decoder_b200 import zmoe_combine, zmoe_get_device_errors
from tests.gpu_util import assert_close, host, require_gpu, to_dev

pytestmark = pytest.mark.gpu


def case(T, d, k, seed, E=16):
    rng = np.random.default_rng(seed)
    if k == 1:
        idx = rng.integers(0, E, size=(T, 1)).astype(np.int32)
    else:
        idx = np.stack([rng.permutation(E)[:2] for _ in range(T)]).astype(np.int32)
    p = oracle.permute(idx, E)
    y_perm = rng.standard_normal((T * k, d)).astype(np.float32)
    gates = rng.uniform(0, 1, size=(T, k)).astype(np.float32)
    res = rng.standard_normal((T, d)).astype(np.float32)
    return p["inv_perm"], y_perm, gates, res


@pytest.mark.parametrize("T,d,k", [(1, 2048, 1), (64, 2048, 1), (1000, 128, 2), (16384, 2048, 2)])
@pytest.mark.parametrize("with_res", [False, True])
def test_combine(T, d, k, with_res):
    require_gpu()
    inv, y_perm, gates, res = case(T, d, k, seed=T + k)
    y = zmoe_combine(to_dev(y_perm, torch.float32), to_dev(inv, torch.int32), to_dev(gates, torch.float32),
                     to_dev(res, torch.float32) if with_res else None)
    want = oracle.combine(y_perm, inv, gates, res if with_res else None)
    assert_close(host(y), want, "f32", "combine")


def test_combine_in_place_residual_and_deterministic():
    require_gpu()
    inv, y_perm, gates, res = case(512, 256, 2, seed=1)
    want = oracle.combine(y_perm, inv, gates, res)
    outs = []
    for _ in range(3):
        h = to_dev(res, torch.float32)
        zmoe_combine(to_dev(y_perm, torch.float32), to_dev(inv, torch.int32), to_dev(gates, torch.float32), h, out=h)
        outs.append(host(h))
    assert_close(outs[0], want, "f32", "in-place combine")
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


def test_combine_bad_row_counts_device_error():
    require_gpu()
    inv, y_perm, gates, _ = case(10, 64, 1, seed=2)
    inv[4, 0] = 10                      # rows are [0, T*k)
    zmoe_get_device_errors()
    y = host(zmoe_combine(to_dev(y_perm, torch.float32), to_dev(inv, torch.int32), to_dev(gates, torch.float32)))
    assert zmoe_get_device_errors() == 1
    assert np.all(y[4] == 0.0)
