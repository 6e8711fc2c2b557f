"""The speaker-embedding prefix row on the GPU vs the oracle (fp32 bar: max |err| <= 1e-4 x RMS; the
products of bf16 weights with fp32 embeddings accumulate in fp32)."""
import numpy as np
import pytest
import torch

import oracle
from moe_inputs import round_to_bf16
from sparse_moe_decoder_b200 import zmoe_speaker_prefix
from tests.gpu_util import TOL, host, rel_err, require_gpu, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("B,d,n_in,dtype,bias", [(1, 2048, 1024, "bf16", True), (3, 2048, 1024, "bf16", False),
                                                 (11, 100, 64, "f32", True), (9, 2050, 1024, "bf16", True)])
def test_speaker_prefix(B, d, n_in, dtype, bias):
    require_gpu()
    rng = np.random.default_rng(B + d)
    W = (rng.standard_normal((d, n_in)) / np.sqrt(n_in)).astype(np.float32)
    if dtype == "bf16":
        W = round_to_bf16(W)
    e = rng.standard_normal((B, n_in)).astype(np.float32)
    b = rng.standard_normal(d).astype(np.float32) if bias else None
    got = zmoe_speaker_prefix(to_dev(e, torch.float32), to_dev(W, torch.bfloat16 if dtype == "bf16" else torch.float32),
                              to_dev(b, torch.float32) if bias else None)
    want = oracle.speaker_prefix(e, W, b)
    assert rel_err(host(got), want) <= TOL["f32"]
