"""Helpers for the GPU parity tests (CUDA path through the C-ABI vs the fp64 oracle)."""
from __future__ import annotations

import numpy as np
import pytest
import torch

# Tolerances of the parity bar: max |gpu - oracle| <= TOL * RMS(oracle output).
TOL = {"bf16": 2e-2, "f32": 1e-4}
# Integer decisions of tokens whose selection margin (from the fp64 oracle) is below this are
# exempt from bit-exact comparison; they are counted and reported.
MARGIN_EXEMPT = 1e-4


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA GPU")


def to_dev(a: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).to(device="cuda", dtype=dtype)


def tdtype(kind: str) -> torch.dtype:
    return torch.bfloat16 if kind == "bf16" else torch.float32


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        t = t.float()
    return t.detach().cpu().numpy()


def rel_err(got: np.ndarray, want: np.ndarray) -> float:
    """max |got - want| / RMS(want)."""
    want = np.asarray(want, np.float64)
    got = np.asarray(got, np.float64)
    if want.size == 0:
        return 0.0
    rms = float(np.sqrt(np.mean(want * want)))
    err = float(np.max(np.abs(got - want)))
    if rms == 0.0:
        return err
    return err / rms


def assert_close(got, want, kind: str, what: str):
    r = rel_err(got, want)
    assert r <= TOL[kind], f"{what}: max|gpu-oracle| = {r:.3e} x RMS > {TOL[kind]:.0e}"
    return r
