"""The N > 1 host path of bench.py on CPU: two gloo ranks, replicas of the
work, job time = the slowest rank's (weak scaling, no data-path collective)."""
import datetime
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


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        mine = 10.0 + 5.0 * rank  # rank 1 is the slow one
        got = bench.max_over_ranks(mine, dist, torch.device("cpu"))
        value = bench.weak_scaling_value(world, 2.0e12, 4, got)
        out.put((rank, got, value))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, got, value in res:
        assert got == 15.0  # both ranks see the slowest rank's time
        assert value == pytest.approx(2 * 2.0e12 * 4 / 15e-3)


def test_single_rank_needs_no_group():
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_value(1, 1e12, 10, 1000.0) == pytest.approx(1e13)
