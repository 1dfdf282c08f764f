"""moe_forward_static: the entry point for callers that cannot allocate device
memory (code inside an allocator or memory-pool callback, a process whose
device memory another runtime has reserved, a plugin handed only its input
and output buffers).  It runs the same kernels on the library's fixed static
scratch instead of a caller workspace, so its output must match moe_forward's
on the same inputs, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import prefill_moe_route_b200 as moe
from checks import bf16_to_f64
from prefill_moe_route_b200.harness import DeviceMoE
from prefill_moe_route_b200.synth import WORKLOADS, Inputs

pytestmark = pytest.mark.gpu


def _within_tol(a_bits, b_bits, atol=2e-2, rtol=2e-2):
    a, b = bf16_to_f64(a_bits), bf16_to_f64(b_bits)
    return bool(np.all(np.abs(a - b) <= atol + rtol * np.abs(b)))


def test_static_scratch_matches_moe_forward_on_consecutive_calls():
    wl = WORKLOADS["decode_tp8"]
    dev = DeviceMoE(wl, Inputs(wl, seed=0))
    out = torch.empty_like(dev.out)
    for call, seed in enumerate((21, 22)):
        inp = Inputs(wl, seed=seed)                      # new tokens and router logits each call
        dev.set_activations(inp.x, inp.logits, inp.bias)
        dev.forward()                                    # caller-owned workspace
        torch.cuda.synchronize()
        want = dev.out_bits().copy()
        out.fill_(0)
        rc = moe.moe_forward_static(dev.shape, dev.x, dev.logits, dev.bias, dev.w13, dev.sf13, dev.w2, dev.sf2,
                                    out, check=False)
        assert rc == moe.MOE_OK, moe.moe_last_error()
        torch.cuda.synchronize()
        got = out.cpu().numpy().view(np.uint16)
        assert _within_tol(got, want), f"call {call}: static-scratch output differs from moe_forward"


def test_static_scratch_rejects_shapes_above_its_size():
    wl = WORKLOADS["prefill_tp4_fp8"]
    t = torch.empty(256, dtype=torch.uint8, device="cuda")   # any device pointers: nothing is launched
    rc = moe.moe_forward_static(wl.shape(), t, t, None, t, t, t, t, t, check=False)
    assert rc == moe.MOE_ERR_WORKSPACE
    assert "static" in moe.moe_last_error()
