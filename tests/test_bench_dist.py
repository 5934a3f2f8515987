"""bench.py's multi-rank arithmetic on CPU: two gloo ranks with different
timings agree on the slowest rank's time, and the job throughput counts the
work of every rank (weak scaling: each rank compresses its own cache)."""
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


def _rank(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        mine = [10.0 + rank, 3.0 - rank, 7.5]
        got = bench.max_over_ranks(mine, dist, "cpu")
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0] == out[1] == [11.0, 3.0, 7.5]


def test_job_throughput_counts_every_rank():
    one = bench.job_gbs(536870912, 1, 1.0)
    assert one == pytest.approx(536.870912)
    assert bench.job_gbs(536870912, 8, 1.0) == pytest.approx(8 * one)
    assert bench.max_over_ranks([1.0, 2.0]) == [1.0, 2.0]   # single process: unchanged
