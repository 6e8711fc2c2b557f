"""The oracle against its pins, and the pins against planted mistakes (CPU only).

A planted mistake is a copy of one oracle function with one plausible error (a
reversed index, a dropped term, a swapped operand, a wrong convention).  Every
such copy must fail at least one pin: otherwise the pins would not be strong
enough to trust the oracle.
"""
import importlib
import math

import numpy as np
import pytest

import oracle
from oracle import delay, embed, ffn, layer
from tests import oracle_pins as P

# the package re-exports a function named ``route``; fetch the module itself
route_mod = importlib.import_module("oracle.route")

GOLDEN_DELAY = P.golden_path("delay_pattern_T4_N3.txt")


# ------------------------------------------------------------------------------------------
# the oracle passes its pins
# ------------------------------------------------------------------------------------------

def test_pin_delay():
    P.pin_delay(oracle.delay_shear, oracle.delay_unshear, GOLDEN_DELAY)


def test_pin_embed():
    P.pin_embed(oracle.embed_sum, oracle.rmsnorm, oracle.embed_sum_rmsnorm)


def test_pin_route():
    P.pin_route(oracle.router_logits, oracle.softmax, oracle.select_topk, oracle.route)


def test_pin_permute():
    P.pin_permute(oracle.permute)


def test_pin_ffn():
    P.pin_ffn(oracle.silu, oracle.swiglu_ffn, oracle.grouped_swiglu)


def test_pin_layer():
    P.pin_layer(oracle.combine, oracle.moe_layer, oracle.moe_layer_bruteforce)


def test_pin_stack():
    P.pin_stack(oracle.decode_stack_step, oracle.embed_sum_rmsnorm, oracle.rmsnorm, oracle.moe_layer_bruteforce)


def test_pin_fp8():
    P.pin_fp8(oracle.e4m3_decode, oracle.dequantize_rows, oracle.moe_layer_fp8)


def test_pin_w8a8():
    P.pin_w8a8(oracle.e4m3_encode, oracle.quantize_rows_dynamic, oracle.moe_layer_w8a8)


def test_pin_speaker():
    P.pin_speaker(oracle.speaker_prefix)


def test_pin_heads():
    P.pin_heads(oracle.head_logits, oracle.greedy, oracle.output_heads, oracle.rmsnorm)


def test_pin_stack_dense():
    P.pin_stack_dense(oracle.decode_stack_step, oracle.embed_sum_rmsnorm, oracle.rmsnorm,
                      oracle.moe_layer_bruteforce)


def test_param_counts_match_published_totals():
    """8B total / 900M active (ZONOS2 Technical Report abstract) at d_model 2048, d_ff 3072."""
    c = oracle.param_counts()
    assert c["experts_total"] == 24 * 16 * 3 * 2048 * 3072 == 7_247_757_312
    assert c["n_moe"] == 24
    assert 7.0e9 <= c["total"] <= 9.0e9, c["total"]
    assert 0.8e9 <= c["active"] <= 1.0e9, c["active"]


# ------------------------------------------------------------------------------------------
# planted mistakes: each one must fail a pin
# ------------------------------------------------------------------------------------------

def _shear_reversed(X, pad):            # Y[t, j] = X[t + j - (N-1), j]: delays run the wrong way
    Xb = np.asarray(X)
    Y = delay.delay_shear(Xb[..., ::-1], pad)[..., ::-1]
    return np.ascontiguousarray(Y)


def _shear_short(X, pad):               # forgets the N - 1 extra rows
    Y = delay.delay_shear(X, pad)
    return Y[..., : np.asarray(X).shape[-2], :]


def _unshear_minus(Y):                  # X_hat[t, j] = Y[t - j, j] (wrong sign)
    Yb = np.asarray(Y)
    squeeze = Yb.ndim == 2
    if squeeze:
        Yb = Yb[None]
    B, Ty, N = Yb.shape
    T = Ty - N + 1
    X = np.empty((B, T, N), np.int32)
    for j in range(N):
        X[:, :, j] = np.roll(Yb[:, :, j], j, axis=1)[:, :T]
    return X[0] if squeeze else X


def _embed_sum_drop_last(ids, tables):
    return embed.embed_sum(np.asarray(ids)[:, :-1], np.asarray(tables)[:-1])


def _rmsnorm_eps_outside(e, gamma, eps):
    e = np.asarray(e, np.float64)
    return e / (np.sqrt(np.mean(e * e, axis=-1, keepdims=True)) + eps) * gamma


def _rmsnorm_no_gamma(e, gamma, eps):
    return embed.rmsnorm(e, np.ones_like(np.asarray(gamma, np.float64)), eps)


def _rmsnorm_no_sqrt(e, gamma, eps):
    e = np.asarray(e, np.float64)
    return e / (np.mean(e * e, axis=-1, keepdims=True) + eps) * gamma


def _route_gate_on_biased(x, W, k, sel_bias=None, logit_bias=None):
    """softmax taken over the selection scores (bias included)."""
    sb = np.zeros(np.asarray(W).shape[0]) if sel_bias is None else np.asarray(sel_bias, np.float64)
    lb = sb if logit_bias is None else sb + np.asarray(logit_bias, np.float64)
    return route_mod.route(x, W, k, sel_bias=None, logit_bias=lb)


def _route_top1_renormalised(x, W, k, sel_bias=None, logit_bias=None):
    sel, g, m, p = route_mod.route(x, W, k, sel_bias, logit_bias)
    return sel, g / g.sum(axis=1, keepdims=True), m, p


def _select_ties_high(s, k):
    s = np.asarray(s, np.float64)
    E = s.shape[1]
    idx = np.broadcast_to(np.arange(E), s.shape)
    return np.lexsort((-idx, -s), axis=-1)[:, :k].astype(np.int32)


def _route_ties_high(x, W, k, sel_bias=None, logit_bias=None):
    orig = route_mod.select_topk
    route_mod.select_topk = _select_ties_high
    try:
        return route_mod.route(x, W, k, sel_bias, logit_bias)
    finally:
        route_mod.select_topk = orig


def _route_margin_top_gap_only(x, W, k, sel_bias=None, logit_bias=None):
    """Planted: the margin is the gap between the two best scores only, whatever k."""
    sel, g, m, p = oracle.route(x, W, k, sel_bias, logit_bias)
    q = oracle.router_logits(x, W) + (0.0 if logit_bias is None else np.asarray(logit_bias))
    s_ = -np.sort(-(q if sel_bias is None else q + np.asarray(sel_bias)), axis=1)
    return sel, g, (s_[:, 0] - s_[:, 1]) if s_.shape[1] > 1 else m, p


def _route_margin_on_logits(x, W, k, sel_bias=None, logit_bias=None):
    """Planted: the margin taken on the unbiased logits instead of the selection scores."""
    sel, g, _, p = oracle.route(x, W, k, sel_bias, logit_bias)
    _, _, m, _ = oracle.route(x, W, k, None, logit_bias)
    return sel, g, m, p


def _permute_descending_t(expert_idx, E, x=None):
    idx = np.asarray(expert_idx)
    T, k = idx.shape
    rev = idx[::-1]
    out = oracle.permute(rev, E, None if x is None else np.asarray(x)[::-1])
    perm = (T - 1 - out["perm"]).astype(np.int32)
    res = dict(out, perm=perm, inv_perm=out["inv_perm"][::-1])
    if x is not None:
        res["x_perm"] = np.asarray(x)[perm]
    return res


def _silu_is_sigmoid(z):
    z = np.asarray(z, np.float64)
    return 1.0 / (1.0 + np.exp(-z))


def _swiglu_swapped(x, wg, wu, wd, return_hidden=False):
    return ffn.swiglu_ffn(x, wu, wg, wd, return_hidden=return_hidden)


def _grouped_off_by_one(x_perm, offsets, wg, wu, wd, experts=None):
    off = np.asarray(offsets).copy()
    off[1:-1] = np.maximum(off[1:-1] - 1, 0)
    return ffn.grouped_swiglu(x_perm, off, wg, wu, wd, experts)


def _combine_no_gate(y_perm, inv_perm, gates, residual=None):
    return layer.combine(y_perm, inv_perm, np.ones_like(np.asarray(gates, np.float64)), residual)


def _combine_no_residual(y_perm, inv_perm, gates, residual=None):
    return layer.combine(y_perm, inv_perm, gates, None)


def _stack_post_norm(ids, tables, gamma0, layers, eps):
    """h <- RMSNorm(h + MoE(h)) instead of h <- h + MoE(RMSNorm(h))."""
    h = embed.embed_sum_rmsnorm(np.atleast_2d(ids), tables, gamma0, eps)
    for L in layers:
        out = layer.moe_layer(h, L["w_router"], None, None, None, L["k"], sel_bias=L["sel_bias"],
                              experts=L["experts"])
        h = embed.rmsnorm(h + out["y"], L["gamma"], eps)
    return dict(h=h, layers=[])


def _stack_dense_no_residual(ids, tables, gamma0, layers, eps):
    """Planted: a dense layer replaces the residual stream instead of adding to it."""
    h = oracle.embed_sum_rmsnorm(np.atleast_2d(ids), tables, gamma0, eps)
    records = []
    for L in layers:
        x = oracle.rmsnorm(h, L["gamma"], eps)
        if L["w_router"] is None:
            h = oracle.swiglu_ffn(x, *L["experts"](0))
            records.append(dict(expert_idx=np.zeros((x.shape[0], 1), np.int64), gates=np.ones((x.shape[0], 1))))
        else:
            out = oracle.moe_layer(x, L["w_router"], None, None, None, L["k"], sel_bias=L["sel_bias"],
                                   experts=L["experts"])
            h = h + out["y"]
            records.append(out)
    return dict(h=h, layers=records)


def _greedy_ties_high(logits):
    """Planted: ties go to the higher id."""
    L = np.asarray(logits)
    return (L.shape[-1] - 1 - np.argmax(L[..., ::-1], axis=-1)).astype(np.int64)


def _heads_margin_top_and_third(h, w_heads, gamma, eps, x_rounded=None):
    """Planted: the heads' margin taken between the largest and the third largest logit."""
    out = oracle.output_heads(h, w_heads, gamma, eps, x_rounded)
    s_ = np.sort(out["logits"], axis=-1)
    out["margin"] = s_[..., -1] - s_[..., -3]
    return out


def _head_logits_transposed(x, w):
    """Planted: the head contracted over the wrong axis of W (rows and columns swapped)."""
    w = np.asarray(w, np.float64)
    return np.einsum("ncv,tc->tnv", w.reshape(w.shape[0], w.shape[2], w.shape[1]), np.asarray(x, np.float64))


def _speaker_transposed(e, w, b=None):
    """Planted: the projection applied with W's axes swapped."""
    e = np.atleast_2d(np.asarray(e, np.float64))
    w = np.asarray(w, np.float64)
    h = e @ w.reshape(w.shape[1], w.shape[0])
    return h + (np.asarray(b, np.float64) if b is not None else 0.0)


def _e4m3_decode_bias8(codes):
    """Planted: exponent bias 8 instead of 7."""
    return oracle.e4m3_decode(codes) / 2.0


def _moe_fp8_scale_per_column(x, w_router, q_gate, s_gate, q_up, s_up, q_down, s_down, k, **kw):
    """Planted: the down projection's scales applied along the contraction (its first f scales) instead
    of along the output rows."""
    deq = lambda q, s: oracle.e4m3_decode(q) * np.asarray(s)[..., None]
    f = q_down.shape[2]
    wd = oracle.e4m3_decode(q_down) * np.resize(np.asarray(s_down), (q_down.shape[0], 1, f))
    return oracle.moe_layer(x, w_router, deq(q_gate, s_gate), deq(q_up, s_up), wd, k, **kw)


def _e4m3_encode_ties_odd(v):
    """Planted: ties go to the odd code."""
    v = np.asarray(v, np.float64)
    q = oracle.e4m3_encode(v).astype(np.int64)
    grid = oracle.e4m3_decode(np.arange(127, dtype=np.uint8))
    a = np.minimum(np.abs(v), 448.0)
    mag = q & 0x7F
    tie = np.zeros(a.shape, bool)
    for c in (mag - 1, mag + 1):
        ok = (c >= 0) & (c <= 126)
        cc = np.clip(c, 0, 126)
        tie |= ok & (np.abs(grid[cc] - a) == np.abs(grid[mag] - a)) & (grid[cc] != grid[mag])
    alt = np.where(np.abs(grid[np.clip(mag + 1, 0, 126)] - a) == np.abs(grid[mag] - a), mag + 1, mag - 1)
    mag = np.where(tie & (mag % 2 == 0), alt, mag)
    return (mag | (q & 0x80)).astype(np.uint8)


def _quantize_per_tensor(a):
    """Planted: one scale for the whole matrix instead of one per token."""
    a32 = np.asarray(a, np.float32)
    amax = np.max(np.abs(a32))
    s = np.float32(amax / np.float32(448.0)) if amax > 0 else np.float32(1.0)
    q = oracle.e4m3_encode((a32 / s).astype(np.float32))
    return q, np.full(a32.shape[:-1], s, np.float32)


def _quantize_by_division(a):
    """Planted: the scaled row formed as row / s instead of row x fp32(1 / s)."""
    a32 = np.asarray(a, np.float32)
    amax = np.max(np.abs(a32), axis=-1)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    return oracle.e4m3_encode((a32 / s[..., None]).astype(np.float32)), s


def _w8a8_layer_with(quantizer):
    import oracle.fp8 as F8
    saved = F8.quantize_rows_dynamic
    def run(*args, **kw):
        F8.quantize_rows_dynamic = quantizer
        try:
            return F8.moe_layer_w8a8(*args, **kw)
        finally:
            F8.quantize_rows_dynamic = saved
    return run


def _w8a8_no_f16_hidden(x, w_router, q_gate, s_gate, q_up, s_up, q_down, s_down, k, **kw):
    """Planted: the hidden activation quantized straight from float64, without its f16 step."""
    x = np.asarray(x, np.float64)
    E = np.asarray(w_router).shape[0]
    sel, gates, _, _ = oracle.route(x, w_router, k, kw.get("sel_bias"), kw.get("logit_bias"))
    p = oracle.permute(sel, E, x)
    qx, sx = oracle.quantize_rows_dynamic(p["x_perm"])
    xq = oracle.e4m3_decode(qx) * sx[:, None].astype(np.float64)
    off = p["offsets"]
    h = np.zeros((xq.shape[0], np.asarray(q_gate).shape[1]))
    y_perm = np.zeros_like(xq)
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            h[a:b] = oracle.silu(xq[a:b] @ oracle.dequantize_rows(q_gate[e], s_gate[e]).T) * \
                (xq[a:b] @ oracle.dequantize_rows(q_up[e], s_up[e]).T)
    qh, sh = oracle.quantize_rows_dynamic(h)
    hq = oracle.e4m3_decode(qh) * sh[:, None].astype(np.float64)
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            y_perm[a:b] = hq[a:b] @ oracle.dequantize_rows(q_down[e], s_down[e]).T
    return dict(y=oracle.combine(y_perm, p["inv_perm"], gates, kw.get("residual")))


MUTANTS = {
    "shear reversed": lambda: P.pin_delay(_shear_reversed, oracle.delay_unshear, GOLDEN_DELAY),
    "shear too short": lambda: P.pin_delay(_shear_short, oracle.delay_unshear, GOLDEN_DELAY),
    "unshear wrong sign": lambda: P.pin_delay(oracle.delay_shear, _unshear_minus, GOLDEN_DELAY),
    "embed drops a codebook": lambda: P.pin_embed(_embed_sum_drop_last, oracle.rmsnorm, oracle.embed_sum_rmsnorm),
    "rmsnorm eps outside root": lambda: P.pin_embed(oracle.embed_sum, _rmsnorm_eps_outside, oracle.embed_sum_rmsnorm),
    "rmsnorm drops gamma": lambda: P.pin_embed(oracle.embed_sum, _rmsnorm_no_gamma, oracle.embed_sum_rmsnorm),
    "rmsnorm drops sqrt": lambda: P.pin_embed(oracle.embed_sum, _rmsnorm_no_sqrt, oracle.embed_sum_rmsnorm),
    "gate on biased scores": lambda: P.pin_route(oracle.router_logits, oracle.softmax, oracle.select_topk,
                                                 _route_gate_on_biased),
    "top-1 gate renormalised": lambda: P.pin_route(oracle.router_logits, oracle.softmax, oracle.select_topk,
                                                   _route_top1_renormalised),
    "ties to the higher index": lambda: P.pin_route(oracle.router_logits, oracle.softmax, _select_ties_high,
                                                    _route_ties_high),
    "margin of the top two scores only": lambda: P.pin_route(oracle.router_logits, oracle.softmax,
                                                             oracle.select_topk, _route_margin_top_gap_only),
    "margin on the unbiased logits": lambda: P.pin_route(oracle.router_logits, oracle.softmax, oracle.select_topk,
                                                         _route_margin_on_logits),
    "permutation not stable": lambda: P.pin_permute(_permute_descending_t),
    "silu is the sigmoid": lambda: P.pin_ffn(_silu_is_sigmoid, oracle.swiglu_ffn, oracle.grouped_swiglu),
    "gate and up swapped": lambda: P.pin_ffn(oracle.silu, _swiglu_swapped, oracle.grouped_swiglu),
    "segment off by one": lambda: P.pin_ffn(oracle.silu, oracle.swiglu_ffn, _grouped_off_by_one),
    "combine ignores gates": lambda: P.pin_layer(_combine_no_gate, oracle.moe_layer, oracle.moe_layer_bruteforce),
    "combine drops residual": lambda: P.pin_layer(_combine_no_residual, oracle.moe_layer,
                                                  oracle.moe_layer_bruteforce),
    "stack post-norm": lambda: P.pin_stack(_stack_post_norm, oracle.embed_sum_rmsnorm, oracle.rmsnorm,
                                           oracle.moe_layer_bruteforce),
    "greedy ties to the higher id": lambda: P.pin_heads(oracle.head_logits, _greedy_ties_high, oracle.output_heads,
                                                         oracle.rmsnorm),
    "heads margin of the top and third logits": lambda: P.pin_heads(oracle.head_logits, oracle.greedy,
                                                                   _heads_margin_top_and_third, oracle.rmsnorm),
    "head contracted on the wrong axis": lambda: P.pin_heads(_head_logits_transposed, oracle.greedy,
                                                              oracle.output_heads, oracle.rmsnorm),
    "e4m3 exponent bias 8": lambda: P.pin_fp8(_e4m3_decode_bias8, oracle.dequantize_rows, oracle.moe_layer_fp8),
    "fp8 down scales per column": lambda: P.pin_fp8(oracle.e4m3_decode, oracle.dequantize_rows,
                                                    _moe_fp8_scale_per_column),
    "speaker projection transposed": lambda: P.pin_speaker(_speaker_transposed),
    "e4m3 ties to the odd code": lambda: P.pin_w8a8(_e4m3_encode_ties_odd, oracle.quantize_rows_dynamic,
                                                    oracle.moe_layer_w8a8),
    "w8a8 activations scaled per tensor": lambda: P.pin_w8a8(oracle.e4m3_encode, oracle.quantize_rows_dynamic,
                                                             _w8a8_layer_with(_quantize_per_tensor)),
    "w8a8 quotient by division": lambda: P.pin_w8a8(oracle.e4m3_encode, _quantize_by_division,
                                                    _w8a8_layer_with(_quantize_by_division)),
    "w8a8 hidden activation without f16": lambda: P.pin_w8a8(oracle.e4m3_encode, oracle.quantize_rows_dynamic,
                                                             _w8a8_no_f16_hidden),
    "dense layer drops residual": lambda: P.pin_stack_dense(_stack_dense_no_residual, oracle.embed_sum_rmsnorm,
                                                            oracle.rmsnorm, oracle.moe_layer_bruteforce),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name):
    with pytest.raises((AssertionError, ValueError, IndexError)):
        MUTANTS[name]()


def test_bruteforce_matches_on_config1_slice():
    """The vectorised layer and the loop layer agree on a slice of the fp32 tiny configuration."""
    from moe_inputs import make_config
    L = make_config(1)
    x = L.x[:6, :16]
    wr = L.w_router[:, :16]
    wg, wu, wd = L.w_gate[:, :8, :16], L.w_up[:, :8, :16], L.w_down[:, :16, :8]
    out = oracle.moe_layer(x, wr, wg, wu, wd, 1, sel_bias=L.sel_bias)
    s, g, y = oracle.moe_layer_bruteforce(x, wr, wg, wu, wd, 1, sel_bias=L.sel_bias)
    assert np.array_equal(out["expert_idx"], s)
    assert np.allclose(out["y"], y, rtol=1e-12, atol=1e-12)
    assert math.isclose(float(np.sum(out["counts"])), 6.0)
