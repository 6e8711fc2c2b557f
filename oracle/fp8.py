"""fp8 expert weights (test infrastructure only: the oracle).

The ZONOS2 serving stack runs the model in fp8 (ZONOS2 page of the sglang-omni cookbook, "Benchmark
Results": the measured serving configuration is fp8).
Reading taken: expert weights stored as E4M3 codes (sign, 4 exponent bits with bias 7, 3 mantissa
bits; exponent field 0 = subnormals m 2^-9; no infinities; 0x7F / 0xFF are NaN) with one fp32 scale
per output row, w = decode(code) * scale.  The decode-size layer is then the bf16 layer's arithmetic on
the decoded weights.  float64.

At prefill sizes the layer runs W8A8 (fp8 weights AND fp8 activations, the scheme fp8 serving stacks
use for dynamic activation quantization): the rows entering each expert GEMM are quantized per token
with a dynamic scale s = max|row| / 448 and codes = the E4M3 value nearest row x (1 / s) (ties to
even, magnitudes saturating at 448); the first GEMM's input is the permuted token row, the second's
the hidden activation h, which is held at 16 bits (f16) between the two GEMMs and quantized from that.
The scale, its reciprocal and the scaled row are computed in fp32 (the precision in which the kernel
takes the same decision: one reciprocal per row, then a multiplication per element, the usual form of
a dynamic-quantization kernel), everything else in float64.
"""
from __future__ import annotations

import numpy as np

from .ffn import silu
from .layer import combine, moe_layer
from .permute import permute
from .route import route


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes (uint8) -> float64 values, from the format's definition."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


def dequantize_rows(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """w = decode(codes) * scale of the row (scales has codes.shape[:-1])."""
    return e4m3_decode(codes) * np.asarray(scales, np.float64)[..., None]


def moe_layer_fp8(x, w_router, q_gate, s_gate, q_up, s_up, q_down, s_down, k, sel_bias=None, logit_bias=None,
                  residual=None) -> dict:
    """One MoE layer whose expert weights are fp8 codes with row scales (router in full precision)."""
    return moe_layer(x, w_router, dequantize_rows(q_gate, s_gate), dequantize_rows(q_up, s_up),
                     dequantize_rows(q_down, s_down), k, sel_bias=sel_bias, logit_bias=logit_bias,
                     residual=residual)


# The 127 non-negative finite E4M3 values, increasing with the code (0x00 .. 0x7E).
_E4M3_GRID = None


def e4m3_encode(v: np.ndarray) -> np.ndarray:
    """Values -> E4M3 codes (uint8): the nearest value of the format's grid, ties to the even code,
    magnitudes beyond 448 saturating to 448; by a nearest-neighbour search over the decoded grid."""
    global _E4M3_GRID
    if _E4M3_GRID is None:
        _E4M3_GRID = e4m3_decode(np.arange(127, dtype=np.uint8))
    v = np.asarray(v, np.float64)
    a = np.minimum(np.abs(v), 448.0)
    i = np.clip(np.searchsorted(_E4M3_GRID, a), 1, 126)          # grid[i - 1] < a <= grid[i]
    lo, hi = _E4M3_GRID[i - 1], _E4M3_GRID[i]
    up = (hi - a < a - lo) | ((hi - a == a - lo) & (i % 2 == 0))  # nearer, or a tie and code i is even
    code = np.where(up, i, i - 1).astype(np.int64)
    code = np.where(a == 0, 0, code)
    return (code | np.where(v < 0, 0x80, 0)).astype(np.uint8)


def quantize_rows_dynamic(a: np.ndarray):
    """Per-row dynamic E4M3 quantization: s = fp32(max|row| / 448) (1 for an all-zero row),
    r = fp32(1 / s) and codes = e4m3_encode(fp32(row x r)).  Returns (codes uint8, s float32)."""
    a32 = np.asarray(a, np.float32)
    amax = np.max(np.abs(a32), axis=-1)
    s = np.where(amax > 0, amax / np.float32(448.0), np.float32(1.0)).astype(np.float32)
    r = (np.float32(1.0) / s).astype(np.float32)
    q = e4m3_encode((a32 * r[..., None]).astype(np.float32))
    return q, s


def moe_layer_w8a8(x, w_router, q_gate, s_gate, q_up, s_up, q_down, s_down, k, sel_bias=None, logit_bias=None,
                   residual=None) -> dict:
    """The MoE layer in W8A8 fp8 (prefill sizes): routing on the unquantized input (router weights in
    full precision), each expert's input rows and hidden rows quantized per token (quantize_rows_dynamic),
    the hidden activation held as f16 before its quantization; fp8 weights with row scales."""
    x = np.asarray(x, np.float64)
    E = np.asarray(w_router).shape[0]
    sel, gates, margin, probs = route(x, w_router, k, sel_bias, logit_bias)
    p = permute(sel, E, x)
    off = p["offsets"]
    qx, sx = quantize_rows_dynamic(p["x_perm"])
    xq = e4m3_decode(qx) * sx[:, None].astype(np.float64)
    M, d = xq.shape
    f = np.asarray(q_gate).shape[1]
    y_perm = np.zeros((M, d))
    h16 = np.zeros((M, f), np.float16)
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b <= a:
            continue
        g = xq[a:b] @ dequantize_rows(q_gate[e], s_gate[e]).T
        u = xq[a:b] @ dequantize_rows(q_up[e], s_up[e]).T
        h16[a:b] = (silu(g) * u).astype(np.float16)
    qh, sh = quantize_rows_dynamic(h16.astype(np.float32))
    hq = e4m3_decode(qh) * sh[:, None].astype(np.float64)
    for e in range(E):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            y_perm[a:b] = hq[a:b] @ dequantize_rows(q_down[e], s_down[e]).T
    y = combine(y_perm, p["inv_perm"], gates, residual)
    return dict(expert_idx=sel, gates=gates, margin=margin, y=y, y_perm=y_perm, h16=h16, qx=qx, sx=sx, qh=qh,
                sh=sh, **p)
