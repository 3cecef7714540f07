"""Multi-process path of bench.py on CPU: N independent replicas (world size
2, gloo), the slowest rank's time, and the whole-job value."""
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
        t = 1.0 + rank                      # rank 1 is the slowest replica
        t_max = bench.max_over_ranks(t, dist, "cpu")
        value = bench.job_value(128 * 10, world, t_max)
        q.put((rank, t_max, value))
    finally:
        dist.destroy_process_group()


def test_replicas_take_the_slowest_rank_and_sum_the_work():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t_max, value in out:
        assert t_max == 2.0
        assert value == pytest.approx(128 * 10 * 2 / 2.0)


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(0.5, None, "cpu") == 0.5
    assert bench.job_value(128, 1, 0.5) == 256
