"""Pins of the fp64 oracle: checks against what the ZONOS2 pages and mathematics fix.

Each ``pin_*`` function takes the oracle function(s) under test as arguments and
raises AssertionError when a pin fails.  ``test_oracle_pins.py`` runs them on the
oracle (they must pass) and on copies with a planted mistake (they must fail).
None of these pins re-types an oracle formula and compares it with itself: they
use hand-worked examples, closed forms, invariants, library routines (torch,
scipy) and pure-Python brute force.
"""
from __future__ import annotations

import math
import os

import numpy as np
import scipy.special
import torch
import torch.nn.functional as F

LOGISTIC_1 = 0.7310585786300049      # 1 / (1 + e^-1), the logistic function at 1
LOGISTIC_M1 = 0.2689414213699951     # 1 / (1 + e^+1)
SILU_2 = 1.7615941559557649          # 2 / (1 + e^-2)


def read_golden_delay(path):
    blocks, cur = {}, None
    with open(path) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            if line.isalpha():
                cur = line
                blocks[cur] = []
                continue
            blocks[cur].append([int(v) for v in line.split()])
    return np.array(blocks["X"], np.int32), np.array(blocks["Y"], np.int32)


# ------------------------------------------------------------------------------------------
# delay pattern
# ------------------------------------------------------------------------------------------

def pin_delay(shear, unshear, golden_path):
    # 1. the hand-worked example
    X, Y = read_golden_delay(golden_path)
    got = shear(X, 1024)
    assert got.shape == Y.shape, (got.shape, Y.shape)
    assert np.array_equal(got, Y), "shear differs from the hand-worked example"
    assert np.array_equal(unshear(Y), X), "unshear differs from the hand-worked example"
    # 2. closed form on X[t, j] = 100 t + j at the pages' N = 9, batched
    B, T, N = 2, 7, 9
    Xc = np.array([[[1000 * b + 100 * t + j for j in range(N)] for t in range(T)] for b in range(B)], np.int32)
    Yc = shear(Xc, -5)
    assert Yc.shape == (B, T + N - 1, N)
    for b in range(B):
        for t in range(T + N - 1):
            for j in range(N):
                want = 1000 * b + 100 * (t - j) + j if 0 <= t - j < T else -5
                assert Yc[b, t, j] == want, (b, t, j, Yc[b, t, j], want)
    # 3. round trip is the identity, including T = 1 and N = 1
    rng = np.random.default_rng(1)
    for (T, N) in [(1, 9), (16, 9), (5, 1), (3, 4)]:
        Xr = rng.integers(0, 1024, size=(T, N)).astype(np.int32)
        assert np.array_equal(unshear(shear(Xr, 1024)), Xr)


# ------------------------------------------------------------------------------------------
# embedding sum + RMSNorm
# ------------------------------------------------------------------------------------------

def pin_embed(embed_sum, rmsnorm, embed_sum_rmsnorm):
    # 1. one-hot tables: table j row v = unit vector at (j + v) mod d, scaled by (j + 1)
    N, V, d = 3, 5, 8
    tab = np.zeros((N, V, d))
    for j in range(N):
        for v in range(V):
            tab[j, v, (j + v) % d] = j + 1
    ids = np.array([[0, 0, 0], [4, 2, 1], [1, 0, 4]])
    want = np.zeros((3, d))
    for t in range(3):
        for j in range(N):
            want[t, (j + ids[t, j]) % d] += j + 1
    assert np.array_equal(embed_sum(ids, tab), want), "embedding sum wrong on one-hot tables"
    # 2. closed-form RMSNorm: e = [3, 4], eps = 0.5 -> mean(e^2) = 12.5, h = e / sqrt(13) * gamma
    e = np.array([[3.0, 4.0]])
    g = np.array([2.0, -1.0])
    h = rmsnorm(e, g, 0.5)
    want = np.array([[6.0 / math.sqrt(13.0), -4.0 / math.sqrt(13.0)]])
    assert np.allclose(h, want, rtol=1e-15, atol=0), (h, want)
    # 3. RMS(h) = 1 exactly (to rounding) when gamma = 1 and eps = 0; scale invariance
    rng = np.random.default_rng(2)
    e = rng.standard_normal((4, 64)) * rng.uniform(0.1, 10, size=(4, 1))
    h = rmsnorm(e, np.ones(64), 0.0)
    assert np.allclose(np.sqrt(np.mean(h * h, axis=1)), 1.0, rtol=1e-14)
    assert np.allclose(rmsnorm(7.5 * e, np.ones(64), 0.0), h, rtol=1e-13)
    # 4. agrees with torch's RMSNorm (library routine) for random gamma and eps
    gamma = rng.standard_normal(64)
    ref = F.rms_norm(torch.from_numpy(e), (64,), weight=torch.from_numpy(gamma), eps=1e-3).numpy()
    assert np.allclose(rmsnorm(e, gamma, 1e-3), ref, rtol=1e-12, atol=1e-13)
    # 5. composition; the zero vector stays zero (eps keeps it finite)
    tab = rng.standard_normal((9, 7, 16))
    ids = rng.integers(0, 7, size=(5, 9))
    gam = rng.standard_normal(16)
    assert np.allclose(embed_sum_rmsnorm(ids, tab, gam, 1e-6), rmsnorm(embed_sum(ids, tab), gam, 1e-6), rtol=1e-14)
    assert np.array_equal(rmsnorm(np.zeros((1, 4)), np.ones(4), 1e-6), np.zeros((1, 4)))


# ------------------------------------------------------------------------------------------
# router
# ------------------------------------------------------------------------------------------

def pin_route(router_logits, softmax, select_topk, route):
    rng = np.random.default_rng(3)
    # 1. logits against torch's linear (library), non-square so a transpose fails
    x = rng.standard_normal((5, 12))
    W = rng.standard_normal((3, 12))
    ref = F.linear(torch.from_numpy(x), torch.from_numpy(W)).numpy()
    assert np.allclose(router_logits(x, W), ref, rtol=1e-13, atol=1e-13)
    # 2. softmax against scipy (library)
    q = rng.standard_normal((6, 16)) * 5
    assert np.allclose(softmax(q), scipy.special.softmax(q, axis=-1), rtol=1e-13, atol=1e-16)
    # 3. hand-worked example: l = [2, 1, 0, 0], b = [0, 1.5, 0, 0] -> s = [2, 2.5, 0, 0]
    e_ = math.e
    W = np.eye(4)
    xr = np.array([[2.0, 1.0, 0.0, 0.0]])
    b = np.array([0.0, 1.5, 0.0, 0.0])
    sel, g, m, p = route(xr, W, 1, sel_bias=b)
    assert sel.tolist() == [[1]]
    # gate is the UNBIASED softmax probability of expert 1, not renormalised
    assert abs(g[0, 0] - e_ / (e_ ** 2 + e_ + 2.0)) < 1e-15, g
    assert abs(m[0] - 0.5) < 1e-15
    sel, g, m, p = route(xr, W, 2, sel_bias=b)
    assert sel.tolist() == [[1, 0]]
    assert abs(g[0, 0] - LOGISTIC_M1) < 1e-15 and abs(g[0, 1] - LOGISTIC_1) < 1e-15, g
    assert abs(m[0] - 0.5) < 1e-15     # min(2.5 - 2, 2 - 0)
    # 4. ties go to the lower index; slot 0 holds the higher score
    s = np.array([[1.0, 3.0, 3.0, 0.0], [0.0, 0.0, 0.0, 0.0], [5.0, 1.0, 5.0, 5.0]])
    assert select_topk(s, 1).tolist() == [[1], [0], [0]]
    assert select_topk(s, 2).tolist() == [[1, 2], [0, 1], [0, 2]]
    # 5. logit_bias shifts both selection and gates: q = l + lb
    lb = np.array([0.0, 0.0, 3.0, 0.0])
    sel, g, m, p = route(xr, W, 1, logit_bias=lb)       # q = [2, 1, 3, 0]
    assert sel.tolist() == [[2]]
    assert abs(g[0, 0] - e_ ** 3 / (e_ ** 2 + e_ + e_ ** 3 + 1.0)) < 1e-15
    # 6. invariants on random inputs
    x = rng.standard_normal((50, 8))
    W = rng.standard_normal((6, 8))
    sel, g, m, p = route(x, W, 1)
    assert np.allclose(g[:, 0], p.max(axis=1), rtol=1e-15)          # b = 0: top-1 gate = max prob
    sel, g, m, p = route(x, W, 2, sel_bias=rng.standard_normal(6))
    assert np.allclose(g.sum(axis=1), 1.0, rtol=1e-14)               # top-2 gates sum to 1
    assert np.all(sel[:, 0] != sel[:, 1])
    # E = 1: the single expert, gate 1
    sel, g, m, p = route(x, W[:1], 1)
    assert np.all(sel == 0) and np.allclose(g, 1.0) and np.all(np.isinf(m))
    # 7. brute force selection on integer scores with many ties
    s = rng.integers(-2, 3, size=(40, 7)).astype(np.float64)
    for k in (1, 2, 3):
        got = select_topk(s, k)
        for t in range(40):
            want = sorted(range(7), key=lambda e: (-s[t, e], e))[:k]
            assert got[t].tolist() == want
    # 8. the margin: hand-worked scores [3, 0.2, 0, -1] (the second gap is the smaller one), on the
    # selection scores (a bias that reorders them moves it), and E = 2 with k = 2 (one gap only)
    xs = np.array([[3.0, 0.2, 0.0, -1.0]])
    m1, m2 = route(xs, np.eye(4), 1)[2][0], route(xs, np.eye(4), 2)[2][0]
    assert abs(m1 - 2.8) < 1e-15 and abs(m2 - 0.2) < 1e-15, (m1, m2)
    m = route(xs, np.eye(4), 2, sel_bias=np.array([0.0, 0.0, 2.5, 0.0]))[2][0]   # s = [3, 0.2, 2.5, -1]
    assert abs(m - 0.5) < 1e-15, m                                               # min(3 - 2.5, 2.5 - 0.2)
    m = route(np.array([[1.0, 4.0]]), np.eye(2), 2)[2][0]
    assert abs(m - 3.0) < 1e-15, m
    # brute force: the smallest gap between consecutive ranks 0..k of the sorted selection scores
    x = rng.standard_normal((30, 6))
    W = rng.standard_normal((5, 6))
    sb = rng.standard_normal(5)
    for k in (1, 2):
        _, _, m, _ = route(x, W, k, sel_bias=sb)
        for t in range(30):
            st = sorted((float(np.dot(W[e], x[t])) + sb[e] for e in range(5)), reverse=True)
            want = min(st[r] - st[r + 1] for r in range(k))
            assert abs(m[t] - want) < 1e-12, (t, k, m[t], want)


# ------------------------------------------------------------------------------------------
# permutation
# ------------------------------------------------------------------------------------------

def pin_permute(permute):
    rng = np.random.default_rng(4)
    for (T, E, k) in [(1, 4, 1), (13, 5, 1), (29, 6, 2), (0, 3, 1), (10, 1, 1)]:
        if k == 2:
            idx = np.stack([rng.permutation(E)[:2] for _ in range(T)]).astype(np.int32)
        else:
            idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
        x = rng.standard_normal((T, 3))
        out = permute(idx, E, x)
        # brute force, in loops
        counts = [0] * E
        for t in range(T):
            for i in range(k):
                counts[idx[t, i]] += 1
        assert out["counts"].tolist() == counts
        offs = [0]
        for c in counts:
            offs.append(offs[-1] + c)
        assert out["offsets"].tolist() == offs
        assert sum(counts) == T * k
        perm, inv = [], {}
        for e in range(E):
            for t in range(T):
                for i in range(k):
                    if idx[t, i] == e:
                        inv[(t, i)] = len(perm)
                        perm.append(t)
        assert out["perm"].tolist() == perm
        for t in range(T):
            for i in range(k):
                assert out["inv_perm"][t, i] == inv[(t, i)]
        for r in range(T * k):
            assert np.array_equal(out["x_perm"][r], x[perm[r]])
    # hand-worked: idx = [2, 0, 2, 1, 0] (k = 1, E = 3)
    out = permute(np.array([[2], [0], [2], [1], [0]], np.int32), 3)
    assert out["counts"].tolist() == [2, 1, 2]
    assert out["offsets"].tolist() == [0, 2, 3, 5]
    assert out["perm"].tolist() == [1, 4, 3, 0, 2]
    assert out["inv_perm"].ravel().tolist() == [3, 0, 4, 2, 1]


# ------------------------------------------------------------------------------------------
# expert FFN
# ------------------------------------------------------------------------------------------

def pin_ffn(silu, swiglu_ffn, grouped_swiglu):
    # 1. textbook values of the logistic function
    z = silu(np.array([0.0, 1.0, -1.0, 2.0]))
    assert np.allclose(z, [0.0, LOGISTIC_1, -LOGISTIC_M1, SILU_2], rtol=1e-15, atol=0)
    # 2. against torch's silu (library) on a wide range, including large |z|
    zz = np.linspace(-60, 60, 1001)
    assert np.allclose(silu(zz), F.silu(torch.from_numpy(zz)).numpy(), rtol=1e-14, atol=1e-300)
    # 3. d = f = 1 hand example: x = 1, W_gate = 1, W_up = 2, W_down = 3 -> y = 3 * silu(1) * 2
    y = swiglu_ffn(np.array([[1.0]]), np.array([[1.0]]), np.array([[2.0]]), np.array([[3.0]]))
    assert abs(y[0, 0] - 6.0 * LOGISTIC_1) < 1e-14, y      # a gate/up swap gives 3 * silu(2)
    # 4. against a composition of torch library ops on random non-square shapes
    rng = np.random.default_rng(5)
    x = rng.standard_normal((7, 6))
    wg, wu, wd = rng.standard_normal((10, 6)), rng.standard_normal((10, 6)), rng.standard_normal((6, 10))
    tx, tg, tu, td = (torch.from_numpy(a) for a in (x, wg, wu, wd))
    ref = F.linear(F.silu(F.linear(tx, tg)) * F.linear(tx, tu), td).numpy()
    y, h = swiglu_ffn(x, wg, wu, wd, return_hidden=True)
    assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)
    assert h.shape == (7, 10)
    # 5. linearity in W_down
    y2 = swiglu_ffn(x, wg, wu, 2.5 * wd)
    assert np.allclose(y2, 2.5 * y, rtol=1e-13)
    # 6. grouped: segments go to their own expert; empty experts allowed
    E = 4
    WG = rng.standard_normal((E, 10, 6))
    WU = rng.standard_normal((E, 10, 6))
    WD = rng.standard_normal((E, 6, 10))
    offsets = np.array([0, 3, 3, 7, 7])
    yp, H = grouped_swiglu(x, offsets, WG, WU, WD)
    for e in range(E):
        a, b = offsets[e], offsets[e + 1]
        if b > a:
            te = [torch.from_numpy(W[e]) for W in (WG, WU, WD)]
            ref = F.linear(F.silu(F.linear(tx[a:b], te[0])) * F.linear(tx[a:b], te[1]), te[2]).numpy()
            assert np.allclose(yp[a:b], ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------------------------------
# combine and the whole layer
# ------------------------------------------------------------------------------------------

def pin_layer(combine, moe_layer, moe_layer_bruteforce):
    # 1. hand-worked combine: 2 tokens, k = 2
    y_perm = np.array([[1.0, 2.0], [10.0, 20.0], [100.0, 200.0], [1000.0, 2000.0]])
    inv = np.array([[0, 3], [2, 1]])
    g = np.array([[0.25, 0.75], [0.5, 0.5]])
    got = combine(y_perm, inv, g, residual=np.array([[1.0, 1.0], [0.0, -1.0]]))
    assert np.allclose(got, [[0.25 + 750.0 + 1.0, 0.5 + 1500.0 + 1.0], [55.0, 109.0]], rtol=1e-15)
    rng = np.random.default_rng(6)
    # 2. brute force on tiny inputs (k = 1 and k = 2, with both biases)
    for k in (1, 2):
        T, d, f, E = 6, 5, 7, 4
        x = rng.standard_normal((T, d))
        wr = rng.standard_normal((E, d))
        wg, wu = rng.standard_normal((E, f, d)), rng.standard_normal((E, f, d))
        wd = rng.standard_normal((E, d, f))
        sb, lb = rng.standard_normal(E), rng.standard_normal(E)
        out = moe_layer(x, wr, wg, wu, wd, k, sel_bias=sb, logit_bias=lb)
        bs, bg, by = moe_layer_bruteforce(x, wr, wg, wu, wd, k, sel_bias=sb, logit_bias=lb)
        assert np.array_equal(out["expert_idx"], bs)
        assert np.allclose(out["gates"], bg, rtol=1e-13)
        assert np.allclose(out["y"], by, rtol=1e-11, atol=1e-12)
        # 3. invariance under a permutation of the tokens
        pi = rng.permutation(T)
        out2 = moe_layer(x[pi], wr, wg, wu, wd, k, sel_bias=sb, logit_bias=lb)
        assert np.allclose(out2["y"], out["y"][pi], rtol=1e-13, atol=1e-14)
        assert np.array_equal(out2["expert_idx"], out["expert_idx"][pi])
    # 4. one expert, top-1 = the dense SwiGLU FFN (torch library ops)
    T, d, f = 9, 6, 11
    x = rng.standard_normal((T, d))
    wg, wu, wd = rng.standard_normal((1, f, d)), rng.standard_normal((1, f, d)), rng.standard_normal((1, d, f))
    out = moe_layer(x, rng.standard_normal((1, d)), wg, wu, wd, 1)
    tx = torch.from_numpy(x)
    ref = F.linear(F.silu(F.linear(tx, torch.from_numpy(wg[0]))) * F.linear(tx, torch.from_numpy(wu[0])),
                   torch.from_numpy(wd[0])).numpy()
    assert np.allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def pin_stack(decode_stack_step, embed_sum_rmsnorm, rmsnorm, moe_layer_bruteforce):
    rng = np.random.default_rng(7)
    N, V, d, f, E = 9, 6, 5, 4, 3
    tables = rng.standard_normal((N, V, d))
    gamma0 = 1 + 0.1 * rng.standard_normal(d)
    ids = rng.integers(0, V, size=(1, N))
    experts = {(l, e): (rng.standard_normal((f, d)), rng.standard_normal((f, d)), rng.standard_normal((d, f)))
               for l in range(3) for e in range(E)}
    layers = []
    for l in range(3):
        layers.append(dict(w_router=rng.standard_normal((E, d)), sel_bias=rng.standard_normal(E),
                           gamma=1 + 0.1 * rng.standard_normal(d), k=2 if l == 2 else 1,
                           experts=(lambda e, l=l: experts[(l, e)])))
    out = decode_stack_step(ids, tables, gamma0, layers, 1e-6)
    # brute force chain: h0 = rmsnorm(sum of 9 rows), then h += moe(rmsnorm(h)) with loop-based layers
    h = embed_sum_rmsnorm(ids, tables, gamma0, 1e-6)
    for l, L in enumerate(layers):
        xin = rmsnorm(h, L["gamma"], 1e-6)
        WG = np.stack([experts[(l, e)][0] for e in range(E)])
        WU = np.stack([experts[(l, e)][1] for e in range(E)])
        WD = np.stack([experts[(l, e)][2] for e in range(E)])
        _, _, y = moe_layer_bruteforce(xin, L["w_router"], WG, WU, WD, L["k"], sel_bias=L["sel_bias"])
        h = h + y
    assert np.allclose(out["h"], h, rtol=1e-12, atol=1e-12)
    # zero down projections: the residual stream is unchanged
    zero = [dict(L, experts=(lambda e, l=l: (experts[(l, e)][0], experts[(l, e)][1], np.zeros((d, f)))))
            for l, L in enumerate(layers)]
    out0 = decode_stack_step(ids, tables, gamma0, zero, 1e-6)
    assert np.allclose(out0["h"], embed_sum_rmsnorm(ids, tables, gamma0, 1e-6), rtol=1e-15)


def pin_stack_dense(decode_stack_step, embed_sum_rmsnorm, rmsnorm, moe_layer_bruteforce):
    """A dense FFN layer (no router) in the stack is h <- h + SwiGLU(RMSNorm(h)), checked against a
    torch composition, followed by a MoE layer checked by the per-token brute force."""
    import torch
    import torch.nn.functional as F
    rng = np.random.default_rng(11)
    N, V, d, f, E = 9, 6, 5, 4, 3
    tables = rng.standard_normal((N, V, d))
    gamma0 = 1 + 0.1 * rng.standard_normal(d)
    ids = rng.integers(0, V, size=(2, N))
    dense = (rng.standard_normal((f, d)), rng.standard_normal((f, d)), rng.standard_normal((d, f)))
    moe = {e: (rng.standard_normal((f, d)), rng.standard_normal((f, d)), rng.standard_normal((d, f))) for e in range(E)}
    g_dense, g_moe = 1 + 0.1 * rng.standard_normal(d), 1 + 0.1 * rng.standard_normal(d)
    w_r, b = rng.standard_normal((E, d)), rng.standard_normal(E)
    layers = [dict(w_router=None, sel_bias=None, gamma=g_dense, k=1, experts=lambda e: dense),
              dict(w_router=w_r, sel_bias=b, gamma=g_moe, k=1, experts=lambda e: moe[e])]
    out = decode_stack_step(ids, tables, gamma0, layers, 1e-6)
    h = embed_sum_rmsnorm(ids, tables, gamma0, 1e-6)
    t = torch.from_numpy(rmsnorm(h, g_dense, 1e-6))
    wg, wu, wd = (torch.from_numpy(w) for w in dense)
    h = h + F.linear(F.silu(F.linear(t, wg)) * F.linear(t, wu), wd).numpy()
    xin = rmsnorm(h, g_moe, 1e-6)
    _, _, y = moe_layer_bruteforce(xin, w_r, np.stack([moe[e][0] for e in range(E)]),
                                   np.stack([moe[e][1] for e in range(E)]), np.stack([moe[e][2] for e in range(E)]),
                                   1, sel_bias=b)
    assert np.allclose(out["h"], h + y, rtol=1e-12, atol=1e-12)
    assert (out["layers"][0]["expert_idx"] == 0).all() and (out["layers"][0]["gates"] == 1).all()


def pin_heads(head_logits, greedy, output_heads, rmsnorm):
    """Heads: one-hot head rows pick coordinates of x (closed form); a brute-force loop; the greedy
    choice on a hand-built example with an exact tie (lower id wins); the pre-norm is RMSNorm."""
    rng = np.random.default_rng(3)
    T, N, V, d = 3, 2, 5, 4
    x = rng.standard_normal((T, d))
    # one-hot rows: logits[t, n, v] = x[t, (n + v) % d]
    W = np.zeros((N, V, d))
    for n in range(N):
        for v in range(V):
            W[n, v, (n + v) % d] = 1.0
    lg = head_logits(x, W)
    for t in range(T):
        for n in range(N):
            for v in range(V):
                assert lg[t, n, v] == x[t, (n + v) % d]
    # brute force on random weights
    W = rng.standard_normal((N, V, d))
    lg = head_logits(x, W)
    for t in range(T):
        for n in range(N):
            for v in range(V):
                acc = 0.0
                for c in range(d):
                    acc += W[n, v, c] * x[t, c]
                assert abs(lg[t, n, v] - acc) <= 1e-12
    # greedy: ties go to the lower id; the maximum wins otherwise
    ex = np.array([[[0.5, 2.0, -1.0, 2.0, 1.9]]])
    assert greedy(ex).tolist() == [[1]]
    assert greedy(-ex).tolist() == [[2]]
    # with a gain the input is the RMSNorm of h; ids are the argmax of its logits
    h = rng.standard_normal((T, d)) * 5.0
    g = 1 + 0.1 * rng.standard_normal(d)
    out = output_heads(h, W, g, 1e-6)
    assert np.allclose(out["x"], rmsnorm(h, g, 1e-6), rtol=1e-15)
    assert np.array_equal(out["ids"], np.argmax(head_logits(rmsnorm(h, g, 1e-6), W), axis=-1))
    assert (out["margin"] >= 0).all()
    # the margin is the gap between the two largest logits: identity head rows make the logits h itself
    out = output_heads(np.array([[0.5, 2.0, -1.0, 1.9], [2.0, 2.0, 0.0, 1.0]]), np.eye(4)[None], None, 1e-6)
    assert out["ids"].tolist() == [[1], [0]]
    assert abs(out["margin"][0, 0] - 0.1) < 1e-15 and out["margin"][1, 0] == 0.0, out["margin"]


def pin_speaker(speaker_prefix):
    """The prefix row is a textbook linear: a hand-worked 2 x 3 example, torch F.linear on random
    non-square weights, and linearity in e."""
    import torch
    import torch.nn.functional as F
    W = np.array([[1.0, 2.0, 3.0], [-1.0, 0.5, 0.0]])
    assert speaker_prefix(np.array([1.0, 1.0, 2.0]), W, np.array([0.5, -0.5])).tolist() == [[9.5, -1.0]]
    rng = np.random.default_rng(4)
    W = rng.standard_normal((7, 11))
    b = rng.standard_normal(7)
    e = rng.standard_normal((3, 11))
    ref = F.linear(torch.from_numpy(e), torch.from_numpy(W), torch.from_numpy(b)).numpy()
    assert np.allclose(speaker_prefix(e, W, b), ref, rtol=1e-12, atol=1e-12)
    e2 = rng.standard_normal((3, 11))
    assert np.allclose(speaker_prefix(e + 2 * e2, W), speaker_prefix(e, W) + 2 * speaker_prefix(e2, W))


def pin_fp8(e4m3_decode, dequantize_rows, moe_layer_fp8):
    """E4M3 decoding: closed forms of the format's corner codes and all 256 codes against torch's
    float8_e4m3fn; a row-scaled 1-expert fp8 layer equals the dense SwiGLU (torch) on w = code * scale."""
    import torch
    import torch.nn.functional as F
    assert e4m3_decode(np.array([0x7E]))[0] == 448.0          # largest finite: 2^8 * 1.75
    assert e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9      # smallest subnormal
    assert e4m3_decode(np.array([0x08]))[0] == 2.0 ** -6      # smallest normal
    assert e4m3_decode(np.array([0x38]))[0] == 1.0
    assert e4m3_decode(np.array([0xC0]))[0] == -2.0
    assert np.isnan(e4m3_decode(np.array([0x7F, 0xFF]))).all()
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    got = e4m3_decode(codes)
    fin = ~np.isnan(ref)
    assert np.array_equal(np.isnan(got), ~fin) and np.array_equal(got[fin], ref[fin])
    rng = np.random.default_rng(8)
    d, f, T = 16, 12, 5
    qg, qu, qd = (rng.integers(0, 0x7F, size=sh).astype(np.uint8) | (rng.integers(0, 2, size=sh) << 7).astype(np.uint8)
                  for sh in ((1, f, d), (1, f, d), (1, d, f)))
    sg, su, sd = rng.random((1, f)) + 0.01, rng.random((1, f)) + 0.01, rng.random((1, d)) + 0.01
    x = rng.standard_normal((T, d))
    out = moe_layer_fp8(x, rng.standard_normal((1, d)), qg, sg, qu, su, qd, sd, 1)
    tg = torch.from_numpy(qg[0]).view(torch.float8_e4m3fn).double() * torch.from_numpy(sg[0])[:, None]
    tu = torch.from_numpy(qu[0]).view(torch.float8_e4m3fn).double() * torch.from_numpy(su[0])[:, None]
    td = torch.from_numpy(qd[0]).view(torch.float8_e4m3fn).double() * torch.from_numpy(sd[0])[:, None]
    tx = torch.from_numpy(x)
    ref = F.linear(F.silu(F.linear(tx, tg)) * F.linear(tx, tu), td).numpy()
    assert np.allclose(out["y"], ref, rtol=1e-12, atol=1e-12)
    assert np.array_equal(dequantize_rows(qg, sg), e4m3_decode(qg) * sg[..., None])


def pin_w8a8(e4m3_encode, quantize_rows_dynamic, moe_layer_w8a8):
    """E4M3 encoding against torch's float8_e4m3fn conversion on the whole grid, every midpoint (ties to
    the even code) and random values, with closed-form ties and saturation; the per-token dynamic scale in
    closed form; a 1-expert W8A8 layer against the same steps written with torch (its float8 and float16
    conversions, F.linear, F.silu)."""
    import torch
    import torch.nn.functional as F
    from oracle import e4m3_decode
    grid = e4m3_decode(np.arange(127, dtype=np.uint8))
    mids = (grid[:-1] + grid[1:]) / 2
    rng = np.random.default_rng(9)
    v = np.concatenate([grid, -grid, mids, -mids, rng.standard_normal(20000) * 40, rng.random(5000) * 2.0 ** -6])
    v32 = v.astype(np.float32)
    ref = torch.from_numpy(v32).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(e4m3_decode(e4m3_encode(v32)), ref)
    assert e4m3_encode(np.array([1.0625]))[0] == 0x38        # tie between 1 (even code) and 1.125
    assert e4m3_encode(np.array([1.1875]))[0] == 0x3A        # tie between 1.125 and 1.25 (even code)
    assert e4m3_encode(np.array([3.0 * 2.0 ** -10]))[0] == 0x02   # subnormal tie 1.5 x 2^-9 -> 2 x 2^-9
    assert list(e4m3_encode(np.array([1000.0, -1000.0, 448.0, 0.0]))) == [0x7E, 0xFE, 0x7E, 0x00]
    row = np.array([[448.0 * 2 ** -3, -2.0 ** -3, 0.5 * 2 ** -3, 0.0]], np.float32)
    q, s = quantize_rows_dynamic(row)
    assert s[0] == np.float32(2 ** -3) and list(q[0]) == [0x7E, 0xB8, 0x30, 0x00]
    q0, s0 = quantize_rows_dynamic(np.zeros((1, 8), np.float32))
    assert s0[0] == 1.0 and not q0.any()
    # the scaled row is row x fp32(1 / s), each product rounded to fp32 (torch's fp32 arithmetic and its
    # float8 conversion): rows with a value next to an E4M3 midpoint, picked where dividing by s instead
    # rounds to the other neighbour
    rows = []
    while len(rows) < 6:
        s_ = np.float32(rng.random() + 0.5)
        amax_ = np.float32(448.0) * s_
        sq = np.float32(amax_ / np.float32(448.0))
        v_ = np.float32(mids[rng.integers(1, 125)] * sq)
        by_mul = np.float32(v_ * np.float32(np.float32(1.0) / sq))
        if e4m3_encode(np.array([by_mul]))[0] != e4m3_encode(np.array([np.float32(v_ / sq)]))[0]:
            rows.append([v_, amax_])
    rows = np.array(rows, np.float32)
    q, s = quantize_rows_dynamic(rows)
    rt = torch.from_numpy(rows)
    st = rt.abs().amax(dim=1) / torch.tensor(448.0, dtype=torch.float32)
    ref_codes = (rt * (1.0 / st)[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(s, st.numpy()) and np.array_equal(q, ref_codes)
    # one expert, W8A8, against torch
    d, f, T = 32, 96, 35     # 3360 hidden values: the f16 step moves ~0.4% of them across an E4M3 midpoint
    qg, qu, qd = (rng.integers(0, 0x7E, size=sh).astype(np.uint8) | (rng.integers(0, 2, size=sh) << 7).astype(np.uint8)
                  for sh in ((1, f, d), (1, f, d), (1, d, f)))
    # row scales of weights whose largest magnitude is ~0.2-0.6 (a 448-code row), tokens of varied size
    sg, su, sd = (((rng.random(sh) + 0.5) * 1e-3).astype(np.float32) for sh in ((1, f), (1, f), (1, d)))
    x = (rng.standard_normal((T, d)) * np.tile([[1.0], [3.0], [0.1], [1e-3], [5.0], [1.0], [2.0]], (5, 1))).astype(np.float32)
    out = moe_layer_w8a8(x, rng.standard_normal((1, d)), qg, sg, qu, su, qd, sd, 1)

    def tq(a32):   # per-row dynamic quantization with torch's conversion, dequantized
        a32 = torch.from_numpy(np.asarray(a32, np.float32))
        s_ = a32.abs().amax(dim=1) / torch.tensor(448.0, dtype=torch.float32)
        s_ = torch.where(s_ > 0, s_, torch.ones_like(s_))
        return (a32 * (1.0 / s_)[:, None]).to(torch.float8_e4m3fn).double() * s_.double()[:, None]

    W = lambda q_, s_: torch.from_numpy(q_[0]).view(torch.float8_e4m3fn).double() * torch.from_numpy(s_[0]).double()[:, None]
    xq = tq(x)
    h = F.silu(F.linear(xq, W(qg, sg))) * F.linear(xq, W(qu, su))
    hq = tq(h.to(torch.float16).float().numpy())
    ref = F.linear(hq, W(qd, sd)).numpy()
    assert np.allclose(out["y"], ref, rtol=1e-12, atol=1e-12)


def golden_path(name):
    return os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", name)
