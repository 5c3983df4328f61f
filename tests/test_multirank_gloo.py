"""The multi-rank host path of bench.py on CPU: two gloo ranks (one process each) run
the same replica bookkeeping the GPU bench runs under torchrun -- a barrier, the
max-over-ranks reduction of the timed region and the whole-job throughput."""
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


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        own_ms = [12.5, 20.0][rank]            # rank 1 is the slow one
        slowest = bench.max_over_ranks_dist(own_ms, world, torch.device("cpu"))
        value = bench.replica_throughput(world, 1000.0, slowest, steps=10)
        results[rank] = (slowest, value)
    finally:
        dist.destroy_process_group()


def test_two_ranks_agree_on_the_slowest_time_and_the_job_throughput():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    results = manager.dict()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert results[0] == results[1]
    slowest, value = results[0]
    assert slowest == 20.0
    # 2 ranks x 1000 units x 10 steps in 20 ms
    assert value == pytest.approx(2 * 1000 * 10 / 0.020)


def test_single_rank_is_identity():
    assert bench.max_over_ranks_dist(3.5, 1, torch.device("cpu")) == 3.5
    assert bench.replica_throughput(1, 100.0, 50.0, 5) == pytest.approx(100 * 5 / 0.05)
