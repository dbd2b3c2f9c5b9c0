"""The multi-rank host logic of bench.py, on CPU with the gloo backend at
world size 2: the step time is the slowest rank's (max over ranks, seen by
every rank), the whole-job throughput counts every rank's bytes, and the
reference arm runs on rank 0 only."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(torch, 1.5 + rank, world, torch.device("cpu"))
        out[rank] = ms
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        port = _free_port()
        procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        assert dict(out) == {0: 2.5, 1: 2.5}


def test_single_rank_and_job_throughput():
    assert bench.max_over_ranks(torch, 3.25, 1, torch.device("cpu")) == 3.25
    # two ranks each streaming 1 GB in 1 ms: 2000 GB/s for the job
    assert bench.job_throughput(2, 1e9, 1.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        steps, warmup, gpus = 1, 1, 2
    assert bench.run_reference(A(), 1, 2) is None
