"""The multi-rank logic of bench.py (one process per GPU, weak scaling) on two
gloo ranks on the CPU: the step time is the max over ranks, each rank draws
its own independent batch, and the whole-job rate counts every rank's work."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        cpu = torch.device("cpu")
        assert bench.dist_env() == (world, rank, rank)
        step_ms = 10.0 + 5.0 * rank  # rank 1 is the slower one
        bench.barrier(cpu)
        worst = bench.max_over_ranks(step_ms, cpu)
        rate = bench.whole_job_rate(1000.0, world, worst * 1e-3)
        seed = bench.shard_seed(1234, rank)
        seeds = [None] * world
        dist.all_gather_object(seeds, seed)
        out[rank] = (worst, rate, seeds)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_time_and_shard_like_the_bench():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        worst, rate, seeds = out[r]
        assert worst == 15.0                      # max over ranks, seen by every rank
        assert rate == pytest.approx(1000.0 * 2 / 0.015)
        assert len(set(seeds)) == world           # independent batches per rank


def test_single_process_helpers_are_identities():
    cpu = torch.device("cpu")
    assert bench.max_over_ranks(3.5, cpu) == 3.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == 5.0
    assert bench.shard_seed(7, 0) == 7
