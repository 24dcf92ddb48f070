"""The bench's multi-GPU form is replicas only: its one collective is the max over ranks of the
timings. Checked here with two gloo ranks on the CPU (no GPU)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    import torch.distributed as dist
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times = [1.0 + rank, 10.0 - rank, 5.0]          # rank 0: [1, 10, 5], rank 1: [2, 9, 5]
        out[rank] = bench.reduce_max_over_ranks(times, dist)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert out[0] == out[1] == [2.0, 10.0, 5.0]


def test_single_rank_and_job_value():
    import bench
    assert bench.reduce_max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
    # two replicas, 1e9 bytes per step each, 10 steps in 100 ms (slowest rank): 200 GB/s
    assert bench.job_value(1e9, 10, 100.0, 2) == pytest.approx(200.0)
