"""moe_forward_static: the entry point for callers that cannot allocate device
memory (code inside an allocator or memory-pool callback, a process whose
device memory another runtime has reserved, a plugin handed only its input
and output buffers).  It runs the same kernels as moe_forward on the library's
fixed static scratch instead of a caller workspace, so its output must be the
same bits as moe_forward's on the same inputs, call after call -- also when
consecutive calls have different shapes (the scratch layout moves with the
shape) and on the grouped kernels.  Device-side timeouts on the static
scratch are reported by moe_get_status_static.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import prefill_moe_route_b200 as moe
from conftest import ROOT
from harness_static import static_call
from prefill_moe_route_b200.harness import DeviceMoE
from prefill_moe_route_b200.synth import WORKLOADS, W_MXFP4, Inputs, Workload

pytestmark = pytest.mark.gpu

MIXED = Workload("static_mixed", 8, 2048, 64, 6, 256, W_MXFP4, 2.5, "normal", True)


def test_static_scratch_matches_moe_forward_bit_for_bit_on_consecutive_calls():
    wl = WORKLOADS["decode_tp8"]
    dev = DeviceMoE(wl, Inputs(wl, seed=0))
    for call, seed in enumerate((21, 22)):
        inp = Inputs(wl, seed=seed)                      # new tokens and router logits each call
        dev.set_activations(inp.x, inp.logits, inp.bias)
        dev.forward()                                    # caller-owned workspace
        torch.cuda.synchronize()
        want = dev.out_bits().copy()
        got = static_call(dev, fill=call + 1)
        rc, st = moe.moe_get_status_static()
        assert rc == moe.MOE_OK and st == 0, (rc, st)
        assert np.array_equal(got, want), f"call {call}: static-scratch output differs from moe_forward"


def test_static_scratch_across_shapes_whose_layouts_differ():
    """decode_tp8, tiny, a third shape, decode_tp8 again: each static call
    clears what its own layout needs and matches moe_forward bit for bit."""
    seq = [WORKLOADS["decode_tp8"], WORKLOADS["tiny"], MIXED, WORKLOADS["decode_tp8"]]
    devs = {}
    for i, wl in enumerate(seq):
        if wl.name not in devs:
            devs[wl.name] = DeviceMoE(wl, Inputs(wl, seed=50 + i))
        dev = devs[wl.name]
        inp = Inputs(wl, seed=60 + i)
        dev.set_activations(inp.x, inp.logits, inp.bias)
        dev.forward()
        torch.cuda.synchronize()
        want = dev.out_bits().copy()
        got = static_call(dev, fill=7)
        assert np.array_equal(got, want), f"step {i} ({wl.name})"


def _child(mode, specs, **env):
    e = dict(os.environ, **{k: str(v) for k, v in env.items()})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "gpu_child.py"), mode, json.dumps(specs)],
                       env=e, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "child ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
    return r.stdout


def test_static_scratch_on_the_grouped_kernels():
    wl = Workload("static_grouped", 8, 1024, 32, 4, 256, W_MXFP4, 2.5, "normal", True)
    spec = [wl.name, wl.M, wl.H, wl.E, wl.topk, wl.I, wl.wfmt, wl.routed_scale, wl.logits, wl.bias]
    out = _child("static_forced_large", [spec], MOE_FORCE_PATH="large")
    assert "ok static forced-large" in out


def test_static_scratch_reports_a_device_timeout():
    wl = Workload("static_withhold", 4, 1024, 32, 4, 256, W_MXFP4, 2.5, "normal", False)
    spec = [wl.name, wl.M, wl.H, wl.E, wl.topk, wl.I, wl.wfmt, wl.routed_scale, wl.logits, wl.bias]
    out = _child("static_withhold", [spec], MOE_TEST_WITHHOLD_FLAG=1, MOE_WAIT_TIMEOUT_MS=20)
    assert "ok static call timed out" in out and "bit-identical" in out


def test_static_scratch_rejects_shapes_above_its_size():
    wl = WORKLOADS["prefill_tp4_fp8"]
    t = torch.empty(256, dtype=torch.uint8, device="cuda")   # any device pointers: nothing is launched
    rc = moe.moe_forward_static(wl.shape(), t, t, None, t, t, t, t, t, check=False)
    assert rc == moe.MOE_ERR_WORKSPACE
    assert "static" in moe.moe_last_error()
