"""The multi-rank legs of bench.py on CPU: two gloo ranks agree on the maximum
of their timings, and the whole-job rate counts every rank's batch over the
slowest rank's time (replicas, weak scaling)."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = [1.0 + rank, 10.0 - rank, 5.0]
        got = bench.max_over_ranks(mine, torch.device("cpu"), world)
        q.put((rank, got))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        assert res[r] == [2.0, 10.0, 5.0]


def test_single_rank_is_identity():
    assert bench.max_over_ranks([3.5, 1.0], torch.device("cpu"), 1) == [3.5, 1.0]


@pytest.mark.parametrize("world", [1, 2, 8])
def test_job_rate_counts_all_ranks(world):
    rate, rate_e2e = bench.job_rates(64, world, 2.0, 4.0)
    assert rate == pytest.approx(64 * world / 2e-3)
    assert rate_e2e == pytest.approx(64 * world / 4e-3)
