"""Summed codebook embeddings and RMSNorm (oracle; test infrastructure only).

Source: ZONOS2 Technical Report digest (audio-paper-digest), "method overview
and architecture", item 5: the decoder input is the sum of the embeddings of the
delayed codebook frame, normalised by RMSNorm before the transformer stack.
RMSNorm itself is the method of "Root Mean Square Layer Normalization", listed
among the works ZONOS2 builds on (ZONOS2 Technical Report, mlsanity.com,
"Builds on").

Readings taken: one table of V = 1025 rows per codebook (ids 0..1023 plus the
pad id 1024, whose row is an ordinary row that is summed like any other);
rmsnorm(e) = e / sqrt(mean(e^2) + eps) * gamma, with eps inside the root.
"""
from __future__ import annotations

import numpy as np


def embed_sum(ids: np.ndarray, tables: np.ndarray) -> np.ndarray:
    """e[t] = sum_j tables[j, ids[t, j]] in float64.  ids [T, N] int, tables [N, V, d]."""
    ids = np.asarray(ids)
    tables = np.asarray(tables)
    T, N = ids.shape
    Nt, V, d = tables.shape
    if Nt != N:
        raise ValueError(f"{N} codebook columns but {Nt} tables")
    if ids.size and (ids.min() < 0 or ids.max() >= V):
        raise ValueError("codebook id outside [0, V)")
    e = np.zeros((T, d), dtype=np.float64)
    for j in range(N):
        e += tables[j, ids[:, j]].astype(np.float64)
    return e


def rmsnorm(e: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """e / sqrt(mean(e^2, last axis) + eps) * gamma, float64."""
    e = np.asarray(e, dtype=np.float64)
    ms = np.mean(e * e, axis=-1, keepdims=True)
    return e / np.sqrt(ms + eps) * np.asarray(gamma, dtype=np.float64)


def embed_sum_rmsnorm(ids: np.ndarray, tables: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """RMSNorm of the summed codebook embeddings: [T, d] float64."""
    return rmsnorm(embed_sum(ids, tables), gamma, eps)
