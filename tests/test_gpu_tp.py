"""The tensor-parallel call on one GPU (needs a B200): the experts' I split
into two 128-aligned slices, each slice's moe_forward_partial run in turn
(what two ranks run at once), the fp32 partials summed (what the all-reduce
does) and rounded by moe_round_bf16; the result matches the oracle's unsplit
call within the parity tolerance, on the single kernel and the grouped
kernels, both weight formats."""
import numpy as np
import pytest
import torch

import oracle
import prefill_moe_route_b200 as moe
from checks import out_within_tol
from prefill_moe_route_b200.synth import W_MXFP4, Workload
from prefill_moe_route_b200.tp import slice_expert_weights
from test_gpu_parity import Problem

pytestmark = pytest.mark.gpu

TP = [Workload("tp_single", 4, 512, 16, 4, 256, W_MXFP4, 2.5, "normal", True),
      Workload("tp_grouped", 40, 512, 16, 4, 256, W_MXFP4, 2.5, "normal", True),
      Workload("tp_grouped_fp8", 40, 384, 16, 3, 256, 2, 2.5, "normal", True)]


@pytest.mark.parametrize("wl", TP, ids=lambda w: w.name)
def test_two_slices_sum_to_the_unsplit_call(wl):
    pb = Problem(wl, seed=71)
    d, world = pb.dev, 2
    sub = dict(wl.shape(), I=wl.I // world)
    partials = []
    for r in range(world):
        w13, s13, w2, s2 = slice_expert_weights(d.w13, d.s13, d.w2, d.s2, wl.wfmt, wl.I, r, world)
        if wl.wfmt == W_MXFP4:   # the kernels read packed MXFP4 scales
            p13, p2 = torch.empty_like(s13), torch.empty_like(s2)
            moe.moe_pack_mxfp4_scales(s13, wl.E, 2 * sub["I"], wl.H, p13)
            moe.moe_pack_mxfp4_scales(s2, wl.E, wl.H, sub["I"], p2)
            s13, s2 = p13, p2
        ws_bytes = moe.moe_workspace_size(sub)
        ws = torch.zeros(ws_bytes, dtype=torch.uint8, device="cuda")
        part = torch.full((wl.M, wl.H), float("nan"), dtype=torch.float32, device="cuda")
        moe.moe_forward_partial(sub, d.x, d.logits, d.bias, w13, s13, w2, s2, part, ws, ws_bytes)
        torch.cuda.synchronize()
        rc, st = moe.moe_get_status(ws)
        assert rc == moe.MOE_OK and st == 0
        assert moe.moe_launches_per_call(sub, 0) == moe.moe_launches_per_call(wl.shape(), 0)   # same path
        partials.append(part)
    total = partials[0] + partials[1]
    out = torch.empty((wl.M, wl.H), dtype=torch.int16, device="cuda")
    moe.moe_round_bf16(total, out, total.numel())
    torch.cuda.synchronize()
    assert np.array_equal(out.cpu().numpy().view(np.uint16),
                          total.cpu().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    ids, tw = oracle.route(pb.inputs.logits, pb.inputs.bias, wl.topk, wl.routed_scale)
    res = oracle.forward_tokens(wl.shape(), pb.inputs.x, ids, tw, *pb.ow)
    ok, worst = out_within_tol(out.cpu().numpy().view(np.uint16), res["ref"])
    assert ok, f"out outside tolerance (worst {worst:.3f} of the bound)"
    # and the partial of the whole I (one rank) is moe_forward's output before rounding
    whole = torch.empty((wl.M, wl.H), dtype=torch.float32, device="cuda")
    moe.moe_forward_partial(wl.shape(), d.x, d.logits, d.bias, d.w13, d.sf13, d.w2, d.sf2, whole, d.workspace,
                            d.ws_bytes)
    d.forward()
    torch.cuda.synchronize()
    assert np.array_equal(d.out_bits(), whole.cpu().to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
