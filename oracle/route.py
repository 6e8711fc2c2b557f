"""Top-k router with a selection-only bias (oracle; test infrastructure only).

Sources:
* ZONOS2 Technical Report digest (audio-paper-digest), "method overview and
  architecture", item 5: 16 experts per MoE layer, top-1 routing, top-2 in the
  last MoE layer.  Item 6: a per-layer bias vector b_l is maintained to push
  expert usage toward uniform.
* "Auxiliary-Loss-Free Load Balancing Strategy for Mixture-of-Experts", listed
  among the works ZONOS2 builds on (ZONOS2 Technical Report, mlsanity.com,
  "Builds on"): the bias shifts which experts are SELECTED, not the gate values.
* The telknet.cc article on ZONOS2, section 2.1 (routing intuition): a linear
  router W_g on the hidden state followed by TopK; the printed equation was lost
  in extraction.

Readings taken (the pages fix none of these):
* logits l = W_r x; q = l + logit_bias (logit_bias is an optional fixed shift
  that affects both selection and gates; the synthetic Zipf skew uses it);
* selection score s = q + b; the k experts with the largest s are chosen,
  ordered by descending s, ties broken toward the lower expert index;
* p = softmax(q) over all E experts (the bias b does not enter);
* k = 1: gate = p[sel_0] (not renormalised);
  k = 2: gate_i = p[sel_i] / (p[sel_0] + p[sel_1]) (renormalised);
* margin (how close the integer decision is to flipping): k = 1:
  s_(1) - s_(2); k = 2: min(s_(1) - s_(2), s_(2) - s_(3)); +inf when there is no
  competitor.
"""
from __future__ import annotations

from typing import Optional

import numpy as np


def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """l[t, e] = sum_c W_r[e, c] x[t, c] in float64."""
    return np.asarray(x, np.float64) @ np.asarray(w_router, np.float64).T


def softmax(q: np.ndarray) -> np.ndarray:
    """exp(q_e - max q) / sum_e' exp(q_e' - max q) along the last axis."""
    q = np.asarray(q, np.float64)
    z = np.exp(q - q.max(axis=-1, keepdims=True))
    return z / z.sum(axis=-1, keepdims=True)


def select_topk(s: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k largest scores per row, by descending score, ties -> lower index."""
    s = np.asarray(s, np.float64)
    T, E = s.shape
    if not 1 <= k <= E:
        raise ValueError(f"k = {k} outside [1, E = {E}]")
    idx = np.broadcast_to(np.arange(E), s.shape)
    order = np.lexsort((idx, -s), axis=-1)   # primary key: -s ascending; secondary: index ascending
    return order[:, :k].astype(np.int32)


def route(x: np.ndarray, w_router: np.ndarray, k: int, sel_bias: Optional[np.ndarray] = None,
          logit_bias: Optional[np.ndarray] = None):
    """Returns (expert_idx int32 [T, k], gates float64 [T, k], margin float64 [T], probs [T, E])."""
    q = router_logits(x, w_router)
    E = q.shape[1]
    if logit_bias is not None:
        q = q + np.asarray(logit_bias, np.float64)[None, :]
    s = q if sel_bias is None else q + np.asarray(sel_bias, np.float64)[None, :]
    sel = select_topk(s, k)
    p = softmax(q)
    rows = np.arange(q.shape[0])[:, None]
    p_sel = p[rows, sel]
    gates = p_sel if k == 1 else p_sel / p_sel.sum(axis=1, keepdims=True)
    # margin on the selection scores, in descending order
    s_sorted = -np.sort(-s, axis=1)
    margin = np.full(q.shape[0], np.inf)
    for r in range(min(k, E - 1)):   # gaps between consecutive ranks 0..k
        margin = np.minimum(margin, s_sorted[:, r] - s_sorted[:, r + 1])
    return sel, gates, margin, p
