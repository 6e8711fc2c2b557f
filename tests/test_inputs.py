"""Seeded input recipes (CPU): the full decoder's FFN stack adds dense layers without moving the
MoE layers' weights."""
import numpy as np

from moe_inputs import StackSpec


def test_full_stack_layout():
    s = StackSpec(d=64, f=64, n_dense_front=3, n_dense_back=1)
    assert s.total_layers == 28
    assert [s.kind(l)[0] for l in (0, 1, 2, 3, 26, 27)] == ["dense", "dense", "dense", "moe", "moe", "dense"]
    assert s.kind(27) == ("dense", 3) and s.kind(3) == ("moe", 0)
    assert [s.k_of(l) for l in range(28)] == [1] * 26 + [2, 1]
    assert [s.E_of(l) for l in (0, 3, 27)] == [1, 16, 1]
    wr, sb, gm = s.layer_small(0)
    assert wr is None and sb is None and gm.shape == (64,)


def test_moe_layers_unchanged_by_dense_layers():
    base = StackSpec(d=64, f=64)
    full = StackSpec(d=64, f=64, n_dense_front=3, n_dense_back=1)
    for m in (0, 23):
        for a, b in zip(base.expert(m, 5), full.expert(3 + m, 5)):
            assert np.array_equal(a, b)
        for a, b in zip(base.layer_small(m), full.layer_small(3 + m)):
            assert np.array_equal(a, b)
    # the dense layers have weights of their own
    assert not np.array_equal(full.expert(0, 0)[0], full.expert(27, 0)[0])
    assert not np.array_equal(full.expert(0, 0)[0], base.expert(0, 0)[0])
