"""The data-parallel plumbing of the multi-GPU path, on two gloo ranks on the CPU.

N GPUs run N replicas (tokens are independent and the weights fit one GPU): every rank takes its
own tokens, and only timings are combined, as the max over ranks (`sparse_moe_decoder_b200.dp`,
used by bench.py under torchrun). Here two processes join a gloo group over 127.0.0.1 and check
that the combination is the element-wise maximum seen by both ranks, that the ranks draw distinct
tokens, and the whole-job rate.
"""
import os
import socket
from datetime import timedelta

import numpy as np
import torch.multiprocessing as mp

from sparse_moe_decoder_b200.dp import job_rate, max_over_ranks, rank_token_seed


def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        # rank r "measured" (1 + r, 10 - r, 5) ms: the slowest rank decides each entry
        got = max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], "cpu")
        # each rank's own tokens (rank 0 keeps the workload's; here every rank draws, for the check)
        x = np.random.default_rng(rank_token_seed(rank)).standard_normal(8)
        q.put((rank, got, x.tolist()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_over_ranks_and_distinct_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(2):
            rank, got, x = q.get(timeout=120)
            results[rank] = (got, x)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    assert results[0][0] == results[1][0] == [2.0, 10.0, 5.0]
    assert not np.allclose(results[0][1], results[1][1])


def test_single_process_and_job_rate():
    # no process group: the values come back unchanged
    assert max_over_ranks([3.5, 1.0]) == [3.5, 1.0]
    # 64 tokens per rank per step, 2 ranks, 10 steps in 1 s (the max over ranks)
    assert job_rate(64, 2, 10, 1000.0) == 1280.0
    assert rank_token_seed(1) != rank_token_seed(2)
