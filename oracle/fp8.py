"""fp8 expert weights (test infrastructure only: the oracle).

The ZONOS2 serving stack runs the model in fp8 (ZONOS2 page of the sglang-omni cookbook, "Benchmark
Results": the measured serving configuration is fp8).
Reading taken: expert weights stored as E4M3 codes (sign, 4 exponent bits with bias 7, 3 mantissa
bits; exponent field 0 = subnormals m 2^-9; no infinities; 0x7F / 0xFF are NaN) with one fp32 scale
per output row, w = decode(code) * scale.  The layer is then the bf16 layer's arithmetic on the
decoded weights.  float64.
"""
from __future__ import annotations

import numpy as np

from .layer import moe_layer


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
