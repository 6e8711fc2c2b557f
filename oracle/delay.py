"""Delay pattern over the RVQ codebooks (oracle; test infrastructure only).

Source: ZONOS2 Technical Report digest (audio-paper-digest), "method overview
and architecture", item 1: with N = 9 DAC codebooks per frame, the model works on
the sheared sequence Y[t, j] = X[t - j, j] (for t >= j), and the inverse
X_hat[t, j] = Y[t + j, j] restores the aligned frames before DAC decoding.

Reading taken where the page is silent: Y has T + N - 1 rows so that every
X[t, j] lands somewhere, and every cell of Y with t - j outside [0, T) holds the
pad id.  This is the only length under which the round trip is the identity.
"""
from __future__ import annotations

import numpy as np


def _as_batched(a: np.ndarray):
    a = np.asarray(a)
    if a.ndim == 2:
        return a[None], True
    if a.ndim == 3:
        return a, False
    raise ValueError(f"expected [T, N] or [B, T, N], got shape {a.shape}")


def delay_shear(X: np.ndarray, pad: int) -> np.ndarray:
    """Y[b, t, j] = X[b, t - j, j] when 0 <= t - j < T, else ``pad``.  Y has T + N - 1 rows."""
    Xb, squeeze = _as_batched(X)
    B, T, N = Xb.shape
    Y = np.full((B, T + N - 1, N), pad, dtype=np.int32)
    for j in range(N):
        # rows t = j .. j + T - 1 of column j receive X[0 .. T - 1, j]
        Y[:, j:j + T, j] = Xb[:, :, j]
    return Y[0] if squeeze else Y


def delay_unshear(Y: np.ndarray) -> np.ndarray:
    """X_hat[b, t, j] = Y[b, t + j, j] for t < T_y - N + 1."""
    Yb, squeeze = _as_batched(Y)
    B, Ty, N = Yb.shape
    T = Ty - N + 1
    if T < 0:
        raise ValueError(f"T_y = {Ty} is shorter than N - 1 = {N - 1}")
    X = np.empty((B, T, N), dtype=np.int32)
    for j in range(N):
        X[:, :, j] = Yb[:, j:j + T, j]
    return X[0] if squeeze else X
