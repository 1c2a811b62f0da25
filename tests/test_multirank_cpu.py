"""The multi-GPU form of the benchmark, checked with two gloo ranks on CPU.

The path has no exchange step, so N GPUs run N independent replicas: each rank
draws its own workload, times its steps, and the job's time is the slowest
rank's. These tests run the same helpers bench.py uses under torchrun."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402

import bench  # noqa: E402
import workloads  # noqa: E402


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workloads.make(1, B=1, H=1, n=256, seed=bench.replica_seed(1, rank))
        own = [1.0 + rank, 10.0 - rank]                   # per-rank step / e2e times (ms)
        mx = bench.max_over_ranks(own, torch, "cpu", world)
        value = bench.job_value(world, 1e9, mx[0])
        dist.barrier()
        q.put((rank, float(wl.q.f64()[0, 0, 0, 0]), mx, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_distinct_replicas():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, x0, mx0, v0), (r1, x1, mx1, v1) = out
    assert mx0 == mx1 == [2.0, 10.0]                       # max over ranks, element-wise
    assert v0 == v1 == pytest.approx(2 * 1e9 / 2.0e-3 / 1e12)  # all ranks' work / slowest time
    assert x0 != x1                                          # each rank has its own replica


def test_single_rank_reduction_is_identity():
    assert bench.max_over_ranks([3.0, 4.0], torch, "cpu", 1) == [3.0, 4.0]
    assert bench.replica_seed(1, 0) == 1001
    assert bench.job_value(1, 2e12, 1000.0) == pytest.approx(2.0)
