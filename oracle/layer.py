"""Combine, the whole MoE layer, and the batch-1 decode stack (oracle; test infrastructure only).

Sources: ZONOS2 Technical Report digest (audio-paper-digest), "method overview
and architecture", item 5 (MoE layers with 16 experts, top-1, top-2 in the last
MoE layer; input = RMSNorm of the summed codebook embeddings) and the telknet.cc
article on ZONOS2, section 2.1 (TopK over router scores; output = gate-weighted
sum of the chosen experts; the printed equation was lost).

moe(x)_t = sum_i gate[t, i] * FFN_{sel[t, i]}(x_t).

Reading taken for the stack (the pages give no per-layer wiring for the FFN
half of a block): pre-norm residual, h <- h + MoE_l(RMSNorm_l(h)), each layer with
its own RMSNorm gain; attention blocks are left out of this path.
"""
from __future__ import annotations

import math
from typing import Callable, Optional, Sequence

import numpy as np

from .embed import embed_sum_rmsnorm, rmsnorm
from .ffn import grouped_swiglu, swiglu_ffn
from .permute import permute
from .route import route


def combine(y_perm: np.ndarray, inv_perm: np.ndarray, gates: np.ndarray,
            residual: Optional[np.ndarray] = None) -> np.ndarray:
    """y[t] = sum_i gates[t, i] * y_perm[inv_perm[t, i]] (+ residual[t]), float64."""
    y_perm = np.asarray(y_perm, np.float64)
    inv = np.asarray(inv_perm)
    g = np.asarray(gates, np.float64)
    T, k = inv.shape
    y = np.zeros((T, y_perm.shape[1]), np.float64)
    for i in range(k):
        y += g[:, i:i + 1] * y_perm[inv[:, i]]
    if residual is not None:
        y += np.asarray(residual, np.float64)
    return y


def moe_layer(x: np.ndarray, w_router: np.ndarray, w_gate, w_up, w_down, k: int,
              sel_bias: Optional[np.ndarray] = None, logit_bias: Optional[np.ndarray] = None,
              residual: Optional[np.ndarray] = None, experts: Optional[Callable] = None) -> dict:
    """One MoE layer: route -> permute -> grouped SwiGLU -> combine.  All intermediates returned."""
    x = np.asarray(x, np.float64)
    E = np.asarray(w_router).shape[0]
    sel, gates, margin, probs = route(x, w_router, k, sel_bias, logit_bias)
    p = permute(sel, E, x)
    y_perm, H = grouped_swiglu(p["x_perm"], p["offsets"], w_gate, w_up, w_down, experts=experts)
    y = combine(y_perm, p["inv_perm"], gates, residual)
    return dict(expert_idx=sel, gates=gates, margin=margin, probs=probs, y_perm=y_perm, H=H, y=y, **p)


def moe_layer_bruteforce(x, w_router, w_gate, w_up, w_down, k, sel_bias=None, logit_bias=None):
    """The same layer as nested pure-Python loops, one token at a time.  Tiny inputs only.

    Shares no helper with the vectorised path: its own dot products, sort, exp.
    Returns (expert_idx [T, k], gates [T, k], y [T, d]) as float lists -> numpy.
    """
    x = np.asarray(x, np.float64)
    W_r = np.asarray(w_router, np.float64)
    Wg = np.asarray(w_gate, np.float64)
    Wu = np.asarray(w_up, np.float64)
    Wd = np.asarray(w_down, np.float64)
    T, d = x.shape
    E, f = Wg.shape[0], Wg.shape[1]
    sel_out = np.zeros((T, k), np.int32)
    gate_out = np.zeros((T, k))
    y_out = np.zeros((T, d))
    for t in range(T):
        q = []
        for e in range(E):
            acc = 0.0
            for c in range(d):
                acc += W_r[e, c] * x[t, c]
            if logit_bias is not None:
                acc += float(logit_bias[e])
            q.append(acc)
        s = [q[e] + (float(sel_bias[e]) if sel_bias is not None else 0.0) for e in range(E)]
        chosen = sorted(range(E), key=lambda e: (-s[e], e))[:k]
        m = max(q)
        z = [math.exp(v - m) for v in q]
        tot = sum(z)
        p = [v / tot for v in z]
        if k == 1:
            g = [p[chosen[0]]]
        else:
            norm = sum(p[e] for e in chosen)
            g = [p[e] / norm for e in chosen]
        for i, e in enumerate(chosen):
            h = []
            for j in range(f):
                a = sum(Wg[e, j, c] * x[t, c] for c in range(d))
                b = sum(Wu[e, j, c] * x[t, c] for c in range(d))
                h.append(a / (1.0 + math.exp(-a)) * b)
            for n in range(d):
                y_out[t, n] += g[i] * sum(Wd[e, n, j] * h[j] for j in range(f))
            sel_out[t, i] = e
            gate_out[t, i] = g[i]
    return sel_out, gate_out, y_out


def decode_stack_step(ids: np.ndarray, tables: np.ndarray, gamma0: np.ndarray,
                      layers: Sequence[dict], eps: float) -> dict:
    """Batch-1 (or batch-T) decode through the MoE stack, float64, no intermediate rounding.

    ``layers[l]`` holds ``w_router``, ``sel_bias``, ``gamma``, ``k`` and ``experts``
    (a callable e -> (W_gate, W_up, W_down)); ``w_router`` None marks a dense FFN layer (expert 0,
    gate 1).  Returns the final h and per-layer records.
    """
    ids = np.atleast_2d(np.asarray(ids))
    h = embed_sum_rmsnorm(ids, tables, gamma0, eps)
    records = []
    for L in layers:
        x = rmsnorm(h, L["gamma"], eps)
        if L["w_router"] is None:
            # a dense FFN layer (ZONOS2 digest item 5: layers 0-2 and 27): the SwiGLU FFN itself
            wg, wu, wd = L["experts"](0)
            y = swiglu_ffn(x, wg, wu, wd)
            out = dict(expert_idx=np.zeros((x.shape[0], 1), np.int64), gates=np.ones((x.shape[0], 1)),
                       margin=np.full(x.shape[0], np.inf), y=y)
        else:
            out = moe_layer(x, L["w_router"], None, None, None, L["k"], sel_bias=L["sel_bias"],
                            experts=L["experts"])
        h = h + out["y"]
        records.append(dict(x=x, expert_idx=out["expert_idx"], gates=out["gates"],
                            margin=out["margin"], y=out["y"], h=h.copy()))
    return dict(h=h, layers=records)
