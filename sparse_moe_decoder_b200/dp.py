"""Data-parallel plumbing for one process per GPU.

Tokens are independent and the weights of the whole stack fit one GPU, so N GPUs run N replicas:
every rank takes its own tokens against replicated weights and no tensor of the data path crosses
GPUs. Only timings are combined, each as the maximum over ranks: a step ends when the slowest rank
ends. Whole-job throughput counts the units every rank processed.
"""
from __future__ import annotations

from typing import Sequence


def rank_token_seed(rank: int) -> int:
    """Seed of rank r's own synthetic tokens (r > 0; rank 0 keeps the workload's tokens)."""
    return 1000 + rank


def max_over_ranks(values: Sequence[float], device="cpu") -> list[float]:
    """Element-wise maximum of `values` over the ranks of the default process group (the values
    themselves when there is no group or a single rank). `device` is where the reduction tensor
    lives: "cuda" for NCCL, "cpu" for gloo."""
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_rate(units_per_rank_step: float, world: int, steps: int, elapsed_ms: float) -> float:
    """Whole-job throughput: the units all `world` ranks processed over `steps` steps, per second of
    the (max-over-ranks) elapsed time."""
    return units_per_rank_step * world * steps / (elapsed_ms / 1e3)
