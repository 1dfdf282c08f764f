"""bench.py's multi-process logic on CPU: world-size-2 gloo process groups
stand in for two GPUs (one replica each).  The timing reduction must take the
slowest rank and report whole-job time per call; the reference arm prints only
on rank 0."""
import contextlib
import io
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from conftest import ROOT

sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, local_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        step_ms, us = bench.whole_job_us_per_call(local_ms[rank], world, dist)
        out[rank] = (step_ms, us)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_whole_job_time_is_the_slowest_rank_over_world_size():
    world, port = 2, _free_port()
    local_ms = [0.050, 0.065]   # rank 1 is slower
    out = mp.Manager().dict()
    mp.spawn(_rank_main, args=(world, port, local_ms, out), nprocs=world, join=True)
    for r in range(world):
        step_ms, us = out[r]
        assert step_ms == pytest.approx(0.065)           # every rank reports the max
        assert us == pytest.approx(0.065 * 1000.0 / 2)   # two calls finish in one slowest step


def test_single_process_is_the_identity():
    assert bench.whole_job_us_per_call(0.04, 1) == (0.04, pytest.approx(40.0))


def test_reference_arm_prints_only_on_rank_zero(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    ns = type("A", (), dict(workload="tiny", steps=1, warmup=0, gpus=2))()
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(ns)
    assert buf.getvalue() == ""
