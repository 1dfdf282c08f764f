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


def test_reference_arm_line_has_the_contract_keys():
    """`bench.py --impl reference` on the host: one JSON line with the
    metric, the reference tag, the oracle baseline and an e2e object."""
    import json
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--workload", "tiny",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, check=True)
    line = json.loads(out.stdout.strip().splitlines()[-1])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["higher_is_better"] is False
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["config"]["workload"].startswith("tiny")


def test_traffic_is_reported_only_for_the_sources_it_was_measured_on(monkeypatch, tmp_path):
    files = ("gemm.cu", "api.cu")
    h = bench._kernel_source_hash(files)
    monkeypatch.setattr(bench, "_NCU_TRAFFIC", {"w": {"gemm1": (files, h, 123)},
                                                "stale": {"gemm1": (files, "0" * 64, 456)}})
    assert bench._traffic("w", "gemm1") == 123
    assert bench._traffic("w", "gemm2") is None
    assert bench._traffic("stale", "gemm1") is None
    assert bench._traffic("absent", "gemm1") is None
    # an edit to one of the kernel's files voids the figure (a copy of the tree, edited)
    import shutil
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(ROOT, "prefill_moe_route_b200", "csrc"), root / "prefill_moe_route_b200" / "csrc")
    shutil.copytree(os.path.join(ROOT, "include"), root / "include")
    with open(root / "prefill_moe_route_b200" / "csrc" / "gemm.cu", "a") as f:
        f.write("// edited\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench._traffic("w", "gemm1") is None


def test_tensor_floor_uses_the_block_scaled_rates():
    from prefill_moe_route_b200.synth import WORKLOADS
    wl = WORKLOADS["decode_tp8"]
    t = bench._tensor_context(wl, 50.0)
    P = wl.M * wl.topk
    assert t["flops"] == pytest.approx(2.0 * P * (2 * wl.I * wl.H + wl.H * wl.I))
    assert 0.0 < t["frac"] < 0.01            # a decode call is nowhere near tensor bound



def test_tensor_floor_takes_each_gemm_kind_from_the_probe():
    """MXFP4 GEMM1 runs kind::mxf4 (the probe's FP4 rate), every other GEMM an
    8-bit kind (its FP8 rate)."""
    from prefill_moe_route_b200.synth import WORKLOADS
    probe = {"fp8": 4000.0, "fp4": 8000.0, "bf16": 2000.0}
    for name, g1_rate in (("prefill_tp8", 8000.0), ("prefill_tp4_fp8", 4000.0)):
        wl = WORKLOADS[name]
        P = wl.M * wl.topk
        f1, f2 = 2.0 * P * 2 * wl.I * wl.H, 2.0 * P * wl.H * wl.I
        t = bench._tensor_context(wl, 1000.0, probe)
        assert t["t_floor_us"] == pytest.approx((f1 / g1_rate + f2 / 4000.0) * 1e-6)
        assert t["frac"] == pytest.approx(t["t_floor_us"] / 1000.0)
        assert "probe" in t["peak_basis"]
