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


def test_e4m3_row_quantizer_matches_torch_and_bounds_the_error():
    import torch
    from moe_inputs import quantize_e4m3_rows
    w = np.random.default_rng(1).standard_normal((4, 33, 50)).astype(np.float32)
    w[0, 0] = 0.0                                     # an all-zero row: scale 1, codes 0
    q, s = quantize_e4m3_rows(w)
    assert q.dtype == np.uint8 and s.shape == (4, 33) and s[0, 0] == 1.0 and not q[0, 0].any()
    tq = (torch.from_numpy(w) / torch.from_numpy(s)[..., None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, tq)
    deq = torch.from_numpy(q).view(torch.float8_e4m3fn).double().numpy() * s[..., None]
    # half a unit in the last place of the code's binade (3 mantissa bits), times the row scale
    assert (np.abs(deq - w) <= np.abs(w) * 2.0 ** -4 + s[..., None] * 2.0 ** -10 + 1e-12).all()
    assert np.allclose(np.max(np.abs(deq), axis=-1)[s != 1.0], np.max(np.abs(w), axis=-1)[s != 1.0], rtol=1e-6)
