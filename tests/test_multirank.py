"""The multi-GPU bench path on CPU: world-size-2 gloo ranks (no GPU).

bench.py runs one independent replica of the workload per GPU (the decode path partitions
over (batch, kv-head) units with no exchange); the only cross-rank steps are the barriers
around the timed region and the maximum of the per-rank times. These tests run those steps
with the gloo backend, and check that the reference arm does its work on rank 0 only.
"""
from __future__ import annotations

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


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        mx = bench.max_over_ranks(times[rank], torch.device("cpu"))
        rate = bench.whole_job_rate(100, world, mx)
        dist.barrier()
        out[rank] = (mx, rate)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_rate_gloo_world2():
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        times = [12.5, 20.0]
        port = _free_port()
        procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=120)
            assert p.exitcode == 0
        for r in range(2):
            mx, rate = out[r]
            assert mx == 20.0  # every rank sees the slowest rank's time
            assert rate == pytest.approx(2 * 100 / 0.020)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.whole_job_rate(10, 1, 5.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank0_only():
    class A:
        steps, warmup, gpus = 1, 3, 2
    # a non-zero rank returns at once, doing no work and printing nothing
    assert bench.run_reference(A(), rank=1) is None
