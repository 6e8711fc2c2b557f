"""Token permutation (dispatch) for grouped experts (oracle; test infrastructure only).

The pages do not describe a dispatch step; it follows from sparse experts
(ZONOS2 Technical Report digest, "method overview and architecture", item 5:
each token visits only its top-k of 16 experts).  Definition used:

* counts[e]  = number of (t, i) with expert_idx[t, i] == e;
* offsets    = exclusive prefix sum of counts, length E + 1;
* rows are ordered by expert ascending, then token ascending (stable);
  perm[row] = t of that row;
* inv_perm[t, i] = the row that holds assignment (t, i);
* x_perm[row] = x[perm[row]].
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def permute(expert_idx: np.ndarray, E: int, x: Optional[np.ndarray] = None):
    """Returns dict(counts, offsets, perm, inv_perm, x_perm)."""
    idx = np.asarray(expert_idx)
    T, k = idx.shape
    flat = idx.reshape(-1)                        # assignment a = t * k + i, t-major
    if flat.size and (flat.min() < 0 or flat.max() >= E):
        raise ValueError("expert index outside [0, E)")
    counts = np.bincount(flat, minlength=E).astype(np.int32) if flat.size else np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    # stable sort by expert keeps ascending assignment index, hence ascending t, inside an expert
    order = np.argsort(flat, kind="stable")
    perm = (order // k).astype(np.int32)
    inv = np.empty(T * k, dtype=np.int32)
    inv[order] = np.arange(T * k, dtype=np.int32)
    out = dict(counts=counts, offsets=offsets, perm=perm, inv_perm=inv.reshape(T, k))
    if x is not None:
        out["x_perm"] = np.asarray(x)[perm]
    return out
