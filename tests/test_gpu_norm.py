"""Embedding sum + RMSNorm and row RMSNorm on the GPU vs the oracle."""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import CODEBOOK_SIZE, PAD_ID, StackSpec, make_codes, round_to_bf16
from sparse_moe_decoder_b200 import zmoe_embed_sum_rmsnorm, zmoe_get_device_errors, zmoe_rmsnorm
from tests.gpu_util import assert_close, host, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,out_kind", [("bf16", "bf16"), ("bf16", "f32"), ("f32", "f32")])
@pytest.mark.parametrize("T", [1, 3, 77])
def test_embed_sum_rmsnorm(kind, out_kind, T):
    require_gpu()
    N, V, d = 9, 1025, 2048
    rng = np.random.default_rng(T)
    tables = rng.standard_normal((N, V, d), dtype=np.float32)
    if kind == "bf16":
        tables = round_to_bf16(tables)
    gamma = (1 + 0.1 * rng.standard_normal(d)).astype(np.float32)
    ids = make_codes(T, N, seed=T)
    ids[0, 3] = PAD_ID                       # the pad row is an ordinary row
    want = oracle.embed_sum_rmsnorm(ids, tables, gamma, 1e-6)
    dt = torch.bfloat16 if kind == "bf16" else torch.float32
    odt = torch.bfloat16 if out_kind == "bf16" else torch.float32
    got = zmoe_embed_sum_rmsnorm(to_dev(ids, torch.int32), to_dev(tables, dt), to_dev(gamma, torch.float32), 1e-6,
                                 out_dtype=odt)
    # the output dtype decides the tolerance (its rounding is part of the result)
    assert_close(host(got), want, "bf16" if out_kind == "bf16" else "f32", "embed_sum_rmsnorm")


def test_embed_one_hot_closed_form():
    """One-hot tables: e has a closed form, RMS(h) = 1 exactly when gamma = 1 (f32 path)."""
    require_gpu()
    N, V, d = 9, 1025, 64
    tables = np.zeros((N, V, d), np.float32)
    for j in range(N):
        tables[j, :, j] = 1.0                 # every row of table j is the unit vector e_j
    ids = make_codes(4, N, seed=1)
    got = host(zmoe_embed_sum_rmsnorm(to_dev(ids, torch.int32), to_dev(tables, torch.float32),
                                      torch.ones(d, device="cuda"), 0.0, out_dtype=torch.float32))
    want = np.zeros((4, d))
    want[:, :N] = np.sqrt(d / N)
    assert np.allclose(got, want, rtol=1e-6)


def test_bad_id_counts_device_error():
    require_gpu()
    N, V, d = 9, 1025, 64
    rng = np.random.default_rng(2)
    tables = rng.standard_normal((N, V, d), dtype=np.float32)
    ids = make_codes(2, N, seed=3)
    ids[1, 4] = CODEBOOK_SIZE + 7            # outside [0, V)
    zmoe_get_device_errors()
    got = host(zmoe_embed_sum_rmsnorm(to_dev(ids, torch.int32), to_dev(tables, torch.float32),
                                      torch.ones(d, device="cuda"), 1e-6, out_dtype=torch.float32))
    assert zmoe_get_device_errors() == 1
    # the bad id contributes nothing; the rest of the row is normalised as usual
    keep = np.ones(N, bool)
    keep[4] = False
    e = tables[np.arange(N)[keep], ids[1][keep]].sum(0).astype(np.float64)
    want = oracle.rmsnorm(e[None], np.ones(d), 1e-6)
    assert np.allclose(got[1], want[0], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("in_kind,out_kind", [("f32", "bf16"), ("f32", "f32"), ("bf16", "bf16")])
def test_rmsnorm_rows(in_kind, out_kind):
    require_gpu()
    rng = np.random.default_rng(9)
    h = (rng.standard_normal((33, 2048)) * rng.uniform(0.1, 30, size=(33, 1))).astype(np.float32)
    if in_kind == "bf16":
        h = round_to_bf16(h)
    gamma = (1 + 0.1 * rng.standard_normal(2048)).astype(np.float32)
    got = zmoe_rmsnorm(to_dev(h, torch.bfloat16 if in_kind == "bf16" else torch.float32),
                       to_dev(gamma, torch.float32), 1e-6,
                       out_dtype=torch.bfloat16 if out_kind == "bf16" else torch.float32)
    assert_close(host(got), oracle.rmsnorm(h, gamma, 1e-6), out_kind, "rmsnorm")


def test_stack_embedding_config5_shapes():
    """The embedding of the batch-1 stack with its own tables and gain (one step)."""
    require_gpu()
    spec = StackSpec()
    tables = spec.tables()
    g0 = spec.gamma0()
    ids = spec.codes(3)
    got = zmoe_embed_sum_rmsnorm(to_dev(ids, torch.int32), to_dev(tables, torch.bfloat16), to_dev(g0, torch.float32),
                                 spec.eps, out_dtype=torch.float32)
    assert_close(host(got), oracle.embed_sum_rmsnorm(ids, tables, g0, spec.eps), "f32", "config-5 embedding")
