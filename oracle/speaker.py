"""Speaker-embedding prefix row (test infrastructure only: the oracle).

ZONOS2 Technical Report digest, "method overview and architecture", item 3 (speaker conditioning):
an ECAPA-TDNN speaker embedding is reduced by LDA to 1024 values e and projected to the model width,
h_spk = W_spk e + b_spk, and the row is prepended to the decoder input as position 0.  The ECAPA and
LDA stages need trained weights and are not part of this path; e is the input here.  float64.
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def speaker_prefix(e: np.ndarray, w_spk: np.ndarray, b_spk: Optional[np.ndarray] = None) -> np.ndarray:
    """h_spk[b] = W_spk e[b] + b_spk: e [B, 1024], W_spk [d, 1024], b_spk [d] -> [B, d] float64."""
    e = np.atleast_2d(np.asarray(e, np.float64))
    h = e @ np.asarray(w_spk, np.float64).T
    if b_spk is not None:
        h = h + np.asarray(b_spk, np.float64)
    return h
