"""More parity cases through the C ABI (needs a B200): an M sweep on both
weight formats, the grouped kernels forced at decode sizes, crafted routing
ties, the single-launch kernel's determinism under repeats, changing inputs
and CUDA-graph replay, and bounded device waits made to run out."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import prefill_moe_route_b200 as moe
from conftest import ROOT
from test_gpu_parity import Problem
from prefill_moe_route_b200.synth import W_FP8_BLOCK128, W_MXFP4, Inputs, Workload

pytestmark = pytest.mark.gpu

SWEEP_M = [1, 2, 3, 5, 8, 9, 16, 17, 31, 32, 33, 63, 64, 65, 127, 128, 255, 256, 511, 2048, 3000]


def _sweep_wl(fmt, M):
    if fmt == W_MXFP4:
        return Workload(f"sweep_mx_M{M}", M, 512, 32, 4, 256, W_MXFP4, 2.5, "normal", True)
    return Workload(f"sweep_fp8_M{M}", M, 384, 24, 3, 256, W_FP8_BLOCK128, 2.5, "normal", True)


def _tokens(M, n=48, seed=1):
    if M <= 256:
        return None
    rng = np.random.default_rng(seed + M)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, n - 2, replace=False)])).astype(np.int32)


@pytest.mark.parametrize("M", SWEEP_M)
@pytest.mark.parametrize("fmt", [W_MXFP4, W_FP8_BLOCK128], ids=["mxfp4", "fp8"])
def test_m_sweep(fmt, M):
    """Every pair's routing and sort bit-exact; mid and out on all tokens up to
    M = 256, on 48 sampled tokens above."""
    pb = Problem(_sweep_wl(fmt, M), seed=M)
    pb.run_and_check(tokens=_tokens(M))


def _child(mode, specs, **env):
    e = dict(os.environ, **{k: str(v) for k, v in env.items()})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "gpu_child.py"), mode, json.dumps(specs)],
                       env=e, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0 and "child ok" in r.stdout, r.stdout[-3000:] + r.stderr[-3000:]
    return r.stdout


def _spec(wl):
    return [wl.name, wl.M, wl.H, wl.E, wl.topk, wl.I, wl.wfmt, wl.routed_scale, wl.logits, wl.bias]


def test_decode_sizes_on_the_grouped_kernels():
    """Every decode-sized MXFP4 case, which normally runs as the single
    kernel, also passes on the grouped kernels (MOE_FORCE_PATH=large)."""
    specs = [_spec(_sweep_wl(W_MXFP4, M)) for M in (1, 2, 3, 5, 8, 9, 16)]
    specs.append(_spec(Workload("decode_like", 4, 6144, 64, 8, 256, W_MXFP4, 2.5, "normal", False)))
    out = _child("forced_large", specs, MOE_FORCE_PATH="large")
    assert out.count("ok forced-large") == len(specs)


def test_the_single_kernel_at_its_largest_sizes():
    """Sizes the plan gives to the grouped kernels (M * topk > 64) but the single
    kernel can run (M <= 16, M * topk <= 256), forced onto it: its 12- and
    16-column variants and up to 256 pairs."""
    specs = [_spec(Workload("small_M12_k8", 12, 1024, 64, 8, 256, W_MXFP4, 2.5, "normal", True)),
             _spec(Workload("small_M16_k8", 16, 2048, 64, 8, 512, W_MXFP4, 2.5, "skew16", False)),
             _spec(Workload("small_M16_k16", 16, 512, 32, 16, 256, W_MXFP4, 2.5, "normal", False))]
    out = _child("forced_small", specs, MOE_FORCE_PATH="small")
    assert out.count("ok forced-small") == len(specs)


def test_single_and_grouped_paths_are_both_exercised():
    for M in (1, 9, 16):      # top-4: M * topk <= 64
        assert moe.moe_launches_per_call(_sweep_wl(W_MXFP4, M).shape(), 0) == 1
    for M in (17, 64):
        assert moe.moe_launches_per_call(_sweep_wl(W_MXFP4, M).shape(), 0) > 1
    assert moe.moe_launches_per_call(dict(_sweep_wl(W_MXFP4, 9).shape(), topk=8), 0) > 1   # 72 pairs
    assert moe.moe_launches_per_call(_sweep_wl(W_FP8_BLOCK128, 4).shape(), 0) > 1


@pytest.mark.parametrize("M", [8, 40])
def test_all_equal_logits_take_the_lowest_ids(M):
    """Every score tied: each token selects experts 0..k-1 (ties go to the lower ID)."""
    wl = Workload(f"ties_M{M}", M, 512, 40, 6, 256, W_MXFP4, 2.5, "normal", False)
    pb = Problem(wl, seed=41)
    logits = np.full((M, wl.E), 0.25, np.float32)
    pb.run_and_check(x=pb.inputs.x, logits=logits)
    ids = pb.dev.taps()["topk_ids"]
    assert np.array_equal(ids, np.tile(np.arange(wl.topk, dtype=np.int32), (M, 1)))


@pytest.mark.parametrize("M", [5, 40])
def test_duplicate_logits_with_e_not_a_multiple_of_32(M):
    """E = 40: lanes own uneven expert counts; logit values repeated across
    experts make the selection rounds meet exact ties."""
    wl = Workload(f"dups_M{M}", M, 512, 40, 6, 256, W_MXFP4, 2.5, "normal", True)
    pb = Problem(wl, seed=43)
    rng = np.random.default_rng(43)
    logits = rng.choice(np.array([-1.0, 0.0, 0.5, 0.5, 1.25, 2.0], np.float32), size=(M, wl.E))
    logits[:, 39] = 2.0                                  # the last expert ties the best ones
    pb.run_and_check(x=pb.inputs.x, logits=logits)


def test_single_kernel_repeat_changing_inputs_and_graph_replay():
    """The single-launch kernel: bit-identical repeats, 40 consecutive calls
    with new inputs on one workspace (each checked: stale epochs or flags
    would show), and a CUDA-graph replay equal to the eager call bit for bit."""
    wl = Workload("single_steps", 6, 512, 16, 4, 256, W_MXFP4, 2.5, "normal", True)
    assert moe.moe_launches_per_call(wl.shape(), 0) == 1
    pb = Problem(wl, seed=47)
    first, taps = pb.run_and_check()
    again, taps2 = pb.run_and_check()
    assert np.array_equal(first, again)
    for k in ("midq", "midqs", "sorted_pairs", "inv"):
        assert np.array_equal(taps[k], taps2[k]), k
    for step in range(40):
        inp = Inputs(wl, seed=1000 + step)
        pb.run_and_check(x=inp.x, logits=inp.logits)
    pb.dev.set_activations(pb.inputs.x, pb.inputs.logits, pb.inputs.bias)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pb.dev.forward(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pb.dev.forward()
    for _ in range(3):
        pb.dev.out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(pb.dev.out_bits(), first)


def test_a_withheld_flag_times_out_and_the_next_call_recovers():
    """A mid flag left unpublished (test knob): the waits on it give up after
    MOE_WAIT_TIMEOUT_MS, the call ends, moe_get_status reports
    MOE_ERR_DEVICE_TIMEOUT with the wait site, and the same workspace then
    serves a normal call that matches the oracle.  No trap, no fault."""
    spec = _spec(Workload("withhold", 4, 1024, 32, 4, 256, W_MXFP4, 2.5, "normal", False))
    out = _child("withhold", [spec], MOE_TEST_WITHHOLD_FLAG=1, MOE_WAIT_TIMEOUT_MS=20)
    assert "ok timed out" in out and "ok next call matches the oracle" in out
