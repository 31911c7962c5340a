"""Host logic of the multi-rank benchmark path, on CPU with two gloo ranks:
every rank replicates the workload, timings are reduced as a maximum over
ranks, the whole-job value counts every rank's work, and the reference arm
runs on rank 0 only."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        # rank 1 is the slow one on the first value, rank 0 on the second
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], world, "cpu")
        value = bench.whole_job_tflops(2.0e12, got[0], world)
        dist.barrier()
    finally:
        dist.destroy_process_group()
    q.put((rank, got, value))


def test_max_over_ranks_and_whole_job_value_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        res = dict((r, (g, v)) for r, g, v in (q.get(timeout=120) for _ in procs))
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for r in (0, 1):
        got, value = res[r]
        assert got == [2.0, 10.0, 3.0]
        # two replicas of 2 TFLOP each in the slowest rank's 2 ms
        assert value == pytest.approx(2 * 2.0e12 / 2e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.whole_job_tflops(1e12, 1.0, 1) == pytest.approx(1000.0)


def test_reference_arm_runs_on_rank_zero_only():
    import argparse
    import bench
    ns = argparse.Namespace(workload="tiny", steps=1, warmup=0)
    assert bench.run_reference(ns, rank=1, world=2) is None
