"""Parameter count of the ZONOS2 decoder at the chosen dimensions (oracle; test infrastructure only).

Sources: ZONOS2 Technical Report (mlsanity.com), Abstract: 8B total parameters,
900M active.  ZONOS2 Technical Report digest, "method overview and
architecture", item 5: 28 layers, the first 3 and the last 1 dense, the others
MoE with 16 experts, top-1 routing and top-2 in the last MoE layer; item 1:
N = 9 codebooks; item 3: a 1024 -> d_model speaker projection.

The pages give neither d_model nor d_ff.  This count checks the chosen
d_model = 2048, d_ff = 3072 against the two published totals.  The attention
shape is not on the pages either: q and o projections d x d, k and v
projections d x kv_dim with kv_dim = 512 (grouped-query attention) are assumed.
"""
from __future__ import annotations


def param_counts(d: int = 2048, f: int = 3072, E: int = 16, n_layers: int = 28, n_dense_front: int = 3,
                 n_dense_back: int = 1, n_codebooks: int = 9, vocab_rows: int = 1025, kv_dim: int = 512,
                 spk_dim: int = 1024) -> dict:
    """Total and active parameter counts (weights only; norms and biases are negligible)."""
    n_moe = n_layers - n_dense_front - n_dense_back
    ffn = 3 * d * f                                   # one SwiGLU expert: gate, up, down
    attn = 2 * d * d + 2 * d * kv_dim                 # q, o, k, v
    emb_heads = 2 * n_codebooks * vocab_rows * d      # 9 input tables + 9 output heads
    routers = n_moe * E * d
    spk = spk_dim * d
    dense_ffn = (n_dense_front + n_dense_back) * ffn
    experts_total = n_moe * E * ffn
    # top-1 in every MoE layer except the last, which is top-2
    experts_active = ((n_moe - 1) * 1 + 2) * ffn
    common = n_layers * attn + dense_ffn + emb_heads + routers + spk
    return dict(total=common + experts_total, active=common + experts_active,
                experts_total=experts_total, experts_active=experts_active, n_moe=n_moe)
