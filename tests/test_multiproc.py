"""The benchmark's multi-rank host logic on CPU: two gloo ranks, no GPU.

Each rank runs its own batch (tokens are independent; no collective on the
data path). The only cross-rank step is the reduction of the timed region to
the slowest rank, and the whole-job throughput counts every rank's tokens.
"""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = [12.5, 17.25][rank]
        ms = bench.reduce_max(local_ms, world)
        dist.barrier()
        q.put((rank, ms, bench.whole_job_tokens_s(4096, world, ms / 10)))
    finally:
        dist.destroy_process_group()


def test_two_ranks_take_the_slowest_time_and_count_all_tokens():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=5) for _ in range(2))
    for rank, ms, tok_s in out:
        assert ms == pytest.approx(17.25)
        assert tok_s == pytest.approx(4096 * 2 / (1.725e-3))


def test_single_rank_needs_no_process_group():
    assert bench.reduce_max(3.0, 1) == 3.0
    assert bench.whole_job_tokens_s(1, 1, 0.5) == pytest.approx(2000.0)
