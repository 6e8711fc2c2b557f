"""fp64 CPU oracle of the ZONOS2 sparse MoE feed-forward path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It shares
no code, constants or helpers with the CUDA library; the only module both sides
read is ``moe_inputs`` (seeded random draws, no arithmetic of the method).

Every function is the plain definition of one step, written in numpy float64
(pure-Python loops only in the ``*_bruteforce`` checkers for tiny inputs), with
the passage of the ZONOS2 pages it follows named in its docstring.  Where the
pages are silent or their formula was lost, the reading taken is stated at the
function.

Pins (see ``tests/test_oracle_pins.py``): every function here is checked
against closed forms, textbook/library special cases, invariants or brute force.
No function is "parity unpinned".
"""
from .delay import delay_shear, delay_unshear
from .embed import embed_sum, rmsnorm, embed_sum_rmsnorm
from .route import router_logits, softmax, select_topk, route
from .permute import permute
from .ffn import silu, swiglu_ffn, grouped_swiglu
from .layer import combine, moe_layer, moe_layer_bruteforce, decode_stack_step
from .params import param_counts
from .heads import head_logits, greedy, output_heads
from .speaker import speaker_prefix
from .fp8 import (e4m3_decode, e4m3_encode, dequantize_rows, moe_layer_fp8, moe_layer_w8a8,
                  quantize_rows_dynamic)

__all__ = [
    "delay_shear", "delay_unshear", "embed_sum", "rmsnorm", "embed_sum_rmsnorm",
    "router_logits", "softmax", "select_topk", "route", "permute", "silu", "swiglu_ffn",
    "grouped_swiglu", "combine", "moe_layer", "moe_layer_bruteforce", "decode_stack_step",
    "param_counts", "head_logits", "greedy", "output_heads", "speaker_prefix",
    "e4m3_decode", "e4m3_encode", "dequantize_rows", "moe_layer_fp8", "moe_layer_w8a8",
    "quantize_rows_dynamic",
]
