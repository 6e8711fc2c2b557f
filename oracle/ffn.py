"""Expert feed-forward network: SwiGLU (oracle; test infrastructure only).

Sources: "GLU Variants Improve Transformer", listed among the works ZONOS2 builds
on (ZONOS2 Technical Report, mlsanity.com, "Builds on"), and the telknet.cc
article on ZONOS2, section 2.1, whose routing formula names SiLU (the equation
itself was lost in extraction).

Reading taken: each expert is a bias-free SwiGLU,
    FFN_e(x) = W_down,e (silu(W_gate,e x) * (W_up,e x)),  silu(z) = z / (1 + exp(-z)),
with W_gate, W_up of shape [f, d] and W_down of shape [d, f].
"""
from __future__ import annotations

import numpy as np


def silu(z: np.ndarray) -> np.ndarray:
    """z * logistic(z) = z / (1 + exp(-z)), float64."""
    z = np.asarray(z, np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_ffn(x: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray,
               return_hidden: bool = False):
    """Rows of x [M, d] through one expert.  Returns y [M, d] (and H [M, f] when asked)."""
    x = np.asarray(x, np.float64)
    g = x @ np.asarray(w_gate, np.float64).T
    u = x @ np.asarray(w_up, np.float64).T
    h = silu(g) * u
    y = h @ np.asarray(w_down, np.float64).T
    return (y, h) if return_hidden else y


def grouped_swiglu(x_perm: np.ndarray, offsets: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray,
                   w_down: np.ndarray, experts=None):
    """Rows offsets[e]:offsets[e+1] of x_perm through expert e.  Returns (y_perm, H).

    ``w_gate`` etc. are [E, ...] arrays, or any indexable whose item e is that expert's
    matrix.  ``experts`` (optional) is a callable e -> (W_gate, W_up, W_down) used instead
    of the arrays, so the caller can produce only the experts that rows reach.
    """
    x_perm = np.asarray(x_perm, np.float64)
    M = x_perm.shape[0]
    E = len(offsets) - 1
    f = None
    y_perm = None
    H = None
    for e in range(E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if b <= a:
            continue
        wg, wu, wd = experts(e) if experts is not None else (w_gate[e], w_up[e], w_down[e])
        y_e, h_e = swiglu_ffn(x_perm[a:b], wg, wu, wd, return_hidden=True)
        if y_perm is None:
            f = h_e.shape[1]
            y_perm = np.zeros((M, y_e.shape[1]), np.float64)
            H = np.zeros((M, f), np.float64)
        y_perm[a:b] = y_e
        H[a:b] = h_e
    if y_perm is None:
        d = x_perm.shape[1]
        f = (np.asarray(w_gate[0]).shape[0] if experts is None else experts(0)[0].shape[0])
        y_perm = np.zeros((M, d), np.float64)
        H = np.zeros((M, f), np.float64)
    return y_perm, H
