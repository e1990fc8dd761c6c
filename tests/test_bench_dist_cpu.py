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


def test_reference_arm_prints_the_contract_line():
    """`bench.py --impl reference` times the oracle on the host cores (here on
    the tiny workload, one thread) and prints one JSON line with the fields
    the driver reads."""
    import json
    import subprocess
    import sys
    from pathlib import Path

    root = Path(__file__).resolve().parents[1]
    out = subprocess.run([sys.executable, str(root / "bench.py"), "--impl", "reference",
                          "--workload", "0", "--steps", "2", "--warmup", "3",
                          "--cpu-threads", "1"],
                         cwd=root, capture_output=True, text=True, timeout=300, check=True)
    d = json.loads(out.stdout.strip().splitlines()[-1])
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["cpu_baseline"]["cores"] == 1 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["config"]["io_dtype"] == "fp32"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]


def test_parity_report_error_measures():
    """The parity report's error measures: normwise max error and the 99.9th
    percentile of the elementwise error with a floor at 1e-3 of the largest
    reference value."""
    import numpy as np
    import parity_report

    ref = np.array([1.0, -2.0, 0.0, 4.0])
    got = ref + np.array([0.0, 0.0, 0.004, -0.04])
    normwise, pct = parity_report.errors(got, ref)
    assert abs(normwise - 0.01) < 1e-12
    # elementwise: 0, 0, 0.004 / max(0, 0.004) = 1, 0.04 / 4 = 0.01
    assert abs(pct - np.percentile([0.0, 0.0, 1.0, 0.01], 99.9)) < 1e-12
