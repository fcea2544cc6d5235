"""The multi-GPU bench runs independent replicas (no collective on the data
path); its only cross-rank step is the max-over-ranks timing.  Checked here
with two gloo ranks on the CPU."""
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
        # rank r took (10 + r) ms for the timed steps and (20 - r) ms end to end
        t, e = bench.max_over_ranks([10.0 + rank, 20.0 - rank], world)
        v = bench.job_throughput(1e12, world, 5, t)
        q.put((rank, t, e, v))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_with_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, t, e, v in res:
        assert t == 11.0 and e == 20.0            # the slowest rank decides
        assert v == pytest.approx(1e12 * 2 * 5 / 11e-3 / 1e12)


def test_single_rank_helpers():
    assert bench.max_over_ranks([3.0, 4.0], 1) == [3.0, 4.0]
    assert bench.job_throughput(2e12, 1, 10, 1000.0) == pytest.approx(20.0)
