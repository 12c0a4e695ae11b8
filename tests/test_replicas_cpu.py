"""The N-GPU benchmark path runs independent replicas (the layer has no
exchange step); the only collective is the max-over-ranks of the timings.
Checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r took (r + 1) ms, 10 * (r + 1) ms and 3 ms on its three timers
        got = bench.max_over_ranks([rank + 1.0, 10.0 * (rank + 1), 3.0], world, torch.device("cpu"))
        q.put((rank, got, bench.job_throughput(2e12, world, got[0])))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, thr in res:
        assert got == [2.0, 20.0, 3.0]                 # the slowest replica's times, on every rank
        assert thr == pytest.approx(2e12 * 2 / 2e-3 / 1e12)


def test_single_rank_is_identity():
    assert bench.max_over_ranks([1.5, 2.5], 1, torch.device("cpu")) == [1.5, 2.5]
    assert bench.job_throughput(1e12, 1, 1.0) == pytest.approx(1000.0)
