"""Output heads over the 9 codebooks + greedy choice (test infrastructure only: the oracle).

ZONOS2 Technical Report digest, "method overview and architecture", item 5 (the decoder predicts
the next frame of the 9 delay-patterned DAC codebooks) and item 1 (the codebooks, Y[t+1, n]).
Reading taken where the pages are silent: the final hidden state passes a last RMSNorm with its
own gain (the pre-norm convention of the stack) and is rounded to bf16 like every layer input;
each codebook has its own bias-free linear head W_n [V, d]; the greedy choice is the argmax over
all V rows, ties to the lower id.  float64, no intermediate rounding beyond the stated input one.
"""
from __future__ import annotations

from typing import Optional

import numpy as np

from .embed import rmsnorm


def head_logits(x: np.ndarray, w_heads: np.ndarray) -> np.ndarray:
    """logits[t, n, v] = sum_c w_heads[n, v, c] * x[t, c]: [T, N, V] float64."""
    x = np.asarray(x, np.float64)
    w = np.asarray(w_heads, np.float64)
    return np.einsum("nvc,tc->tnv", w, x)


def greedy(logits: np.ndarray) -> np.ndarray:
    """argmax over the last axis, the lowest index among equal maxima (numpy's argmax rule)."""
    return np.argmax(logits, axis=-1).astype(np.int64)


def output_heads(h: np.ndarray, w_heads: np.ndarray, gamma: Optional[np.ndarray], eps: float,
                 x_rounded: Optional[np.ndarray] = None) -> dict:
    """The heads on the final hidden state h [T, d].  With gamma the input is RMSNorm(h) * gamma.

    ``x_rounded`` lets a caller pass the bf16-rounded input it consumed (the rounding is the one
    step of the path that is not fp64); the logits are then formed from it."""
    x = rmsnorm(h, gamma, eps) if gamma is not None else np.asarray(h, np.float64)
    xin = x if x_rounded is None else np.asarray(x_rounded, np.float64)
    logits = head_logits(xin, w_heads)
    top2 = np.sort(logits, axis=-1)[..., -2:] if logits.shape[-1] > 1 else None
    margin = (top2[..., 1] - top2[..., 0]) if top2 is not None else np.full(logits.shape[:-1], np.inf)
    return dict(x=x, logits=logits, ids=greedy(logits), margin=margin)
