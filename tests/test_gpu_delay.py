"""Delay shear / unshear on the GPU vs the oracle: bit-exact."""
import numpy as np
import pytest

import oracle
from moe_inputs import PAD_ID, config1_codes, make_codes
from sparse_moe_decoder_b200 import zmoe_delay_shear, zmoe_delay_unshear
from tests.gpu_util import host, require_gpu, to_dev

import torch

pytestmark = pytest.mark.gpu


def test_config1_codes_bit_exact():
    require_gpu()
    X = config1_codes()                       # int32 [16, 9]
    Y = zmoe_delay_shear(to_dev(X, torch.int32), PAD_ID)
    torch.cuda.synchronize()
    assert np.array_equal(host(Y), oracle.delay_shear(X, PAD_ID))
    Xh = zmoe_delay_unshear(Y)
    assert np.array_equal(host(Xh), X)


@pytest.mark.parametrize("B,T,N", [(1, 1, 9), (3, 37, 9), (2, 0, 9), (4, 513, 9), (1, 5, 1), (2, 7, 64),
                                   (8, 2048, 9)])
def test_shapes_bit_exact(B, T, N):
    require_gpu()
    X = make_codes(T, N, seed=B * 100 + T, batch=B)
    Y = zmoe_delay_shear(to_dev(X, torch.int32), PAD_ID)
    assert np.array_equal(host(Y), oracle.delay_shear(X, PAD_ID))
    assert np.array_equal(host(zmoe_delay_unshear(Y)), X)


def test_unshear_of_arbitrary_Y():
    """Unshear reads only the diagonal cells; random Y (not produced by shear)."""
    require_gpu()
    rng = np.random.default_rng(5)
    Y = rng.integers(-5, 2000, size=(3, 40, 9)).astype(np.int32)
    assert np.array_equal(host(zmoe_delay_unshear(to_dev(Y, torch.int32))), oracle.delay_unshear(Y))
