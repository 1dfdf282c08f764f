"""Parity of the CUDA path with the oracle, through the C ABI (needs a B200).

Bit-exact: quantized weights, routing ids and weights, the pair sort.
Within one E4M3 step with scales exact (binade-edge blocks counted): mid.
Within 2e-2 absolute + 2e-2 relative of the oracle's fp64 result: bf16 out.
"""
import numpy as np
import pytest
import torch

import oracle
import prefill_moe_route_b200 as moe
from checks import out_within_tol, verify_call
from prefill_moe_route_b200.harness import DeviceMoE
from prefill_moe_route_b200.synth import WORKLOADS, W_MXFP4, Inputs, Workload

pytestmark = pytest.mark.gpu


def _oracle_weight_arrays(wl):
    E, H, I = wl.E, wl.H, wl.I
    if wl.wfmt == W_MXFP4:
        return [np.empty((E, 2 * I, H // 2), np.uint8), np.empty((E, 2 * I, H // 32), np.uint8),
                np.empty((E, H, I // 2), np.uint8), np.empty((E, H, I // 32), np.uint8)]
    return [np.empty((E, 2 * I, H), np.uint8), np.empty((E, 2 * I // 128, H // 128), np.float32),
            np.empty((E, H, I), np.uint8), np.empty((E, H // 128, I // 128), np.float32)]


class Problem:
    """One workload on the GPU plus the oracle's own quantization of the same draws."""

    def __init__(self, wl: Workload, seed: int = 0):
        self.wl = wl
        self.inputs = Inputs(wl, seed)
        self.ow = _oracle_weight_arrays(wl)

        def on_expert(e, f13, f2):
            if wl.wfmt == W_MXFP4:
                q13, s13 = oracle.quant_mxfp4(f13)
                q2, s2 = oracle.quant_mxfp4(f2)
            else:
                q13, s13 = oracle.quant_fp8_block128(f13)
                q2, s2 = oracle.quant_fp8_block128(f2)
            self.ow[0][e], self.ow[1][e], self.ow[2][e], self.ow[3][e] = q13, s13, q2, s2

        self.dev = DeviceMoE(wl, self.inputs, on_expert=on_expert)

    def check_weights(self):
        for g, o in zip(self.dev.weights_host(), self.ow):
            assert g.shape == o.shape
            assert np.array_equal(g.view(np.uint8), o.view(np.uint8))

    def run_and_check(self, tokens=None, x=None, logits=None):
        wl, dev = self.wl, self.dev
        if x is not None:
            dev.set_activations(x, logits, self.inputs.bias)
        else:
            x, logits = self.inputs.x, self.inputs.logits
        dev.forward()
        torch.cuda.synchronize()
        words = dev.status_words()
        rc, st = dev.status()
        assert rc == moe.MOE_OK and st == 0, f"device status {st}, wait site {int(words[2]) & 0xFFFFFFFF:#x}"
        taps = dev.taps()
        verify_call(wl, taps, dev.out_bits(), logits, self.inputs.bias, x, self.ow, tokens=tokens)
        return dev.out_bits().copy(), taps


def _sample(M, n=16, seed=0):
    if M <= n:
        return None
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([[0, M - 1], rng.choice(M, n - 2, replace=False)])).astype(np.int32)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_parity(name):
    wl = WORKLOADS[name]
    pb = Problem(wl)
    pb.check_weights()
    pb.run_and_check(tokens=_sample(wl.M))


def test_decode_with_router_bias():
    pb = Problem(WORKLOADS["decode_tp8"].with_(bias=True), seed=3)
    pb.run_and_check()


SMALL = [
    # ragged token tiles, several tiles per expert, both formats, degenerate routings
    Workload("ragged_mx", 40, 512, 16, 4, 256, 1, 2.5, "normal", True),
    Workload("ragged_fp8", 40, 512, 8, 2, 256, 2, 2.5, "normal", True),
    Workload("two_tiles_mx", 150, 512, 4, 4, 128, 1, 1.0, "normal", False),     # k = E, 150 > 64 rows
    Workload("two_tiles_fp8", 150, 256, 4, 2, 256, 2, 1.0, "skew16", False),
    Workload("dense_mx", 33, 512, 1, 1, 128, 1, 1.0, "normal", False),          # E = k = 1
    Workload("one_token_mx", 1, 1024, 32, 8, 128, 1, 2.5, "normal", True),
    Workload("one_token_fp8", 1, 384, 32, 8, 128, 2, 2.5, "normal", True),
    Workload("mid16_mx", 16, 768, 64, 6, 384, 1, 2.5, "normal", True),
    Workload("mid33_fp8", 33, 640, 64, 6, 384, 2, 2.5, "zipf1.1", False),
    # block-FP8 with >= 32 pairs per expert: 128-pair tiles (the wide kernels);
    # ragged tails, and H = 640 leaves GEMM2's last task with one h-tile
    Workload("wide_fp8", 300, 640, 4, 2, 384, 2, 2.5, "normal", True),
    Workload("wide_fp8_zipf", 640, 512, 16, 4, 256, 2, 2.5, "zipf1.1", False),
    Workload("wide_fp8_one_tile", 65, 256, 2, 2, 128, 2, 1.0, "normal", False),   # k = E: 65 pairs each
    # k = E, M = 192: each expert's second 128-pair tile holds exactly 64 pairs
    Workload("wide_fp8_half_edge", 192, 256, 2, 2, 128, 2, 1.0, "normal", False),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_small_parity(wl):
    pb = Problem(wl, seed=7)
    pb.check_weights()
    pb.run_and_check()


def test_route_entry_point():
    for name in ("tiny", "decode_tp8", "prefill_tp4_fp8"):
        wl = WORKLOADS[name]
        inp = Inputs(wl.with_(bias=True), seed=5)
        logits = torch.from_numpy(inp.logits).cuda()
        bias = torch.from_numpy(inp.bias).cuda()
        ids = torch.empty((wl.M, wl.topk), dtype=torch.int32, device="cuda")
        w = torch.empty((wl.M, wl.topk), dtype=torch.float32, device="cuda")
        moe.moe_route(wl.shape(), logits, bias, ids, w)
        torch.cuda.synchronize()
        rid, rw = oracle.route(inp.logits, inp.bias, wl.topk, wl.routed_scale)
        assert np.array_equal(ids.cpu().numpy(), rid)
        assert np.array_equal(w.cpu().numpy().view(np.uint32), rw.view(np.uint32))


def test_determinism_changing_inputs_and_graph_replay():
    wl = Workload("steps", 24, 512, 16, 4, 256, 1, 2.5, "normal", True)
    pb = Problem(wl, seed=11)
    first, taps = pb.run_and_check()
    again, taps2 = pb.run_and_check()
    assert np.array_equal(first, again) and np.array_equal(taps["midq"], taps2["midq"])
    # consecutive calls with new activations on one workspace, each checked
    for step in range(12):
        inp = Inputs(wl, seed=100 + step)
        pb.run_and_check(x=inp.x, logits=inp.logits)
    # a CUDA-graph replay gives the eager result bit for bit
    pb.dev.set_activations(pb.inputs.x, pb.inputs.logits, pb.inputs.bias)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        pb.dev.forward(stream=s)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pb.dev.forward()
    pb.dev.out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert np.array_equal(pb.dev.out_bits(), first)


def test_error_codes_on_device():
    wl = WORKLOADS["tiny"]
    pb = Problem(wl)
    d = pb.dev
    rc = moe.moe_forward(d.shape, d.x, d.logits, d.bias, d.w13, d.sf13, d.w2, d.sf2, d.out, d.workspace,
                         d.ws_bytes - 256, check=False)
    assert rc == moe.MOE_ERR_WORKSPACE
    host = torch.empty(16, dtype=torch.int32)
    rc = moe.moe_forward(d.shape, host.data_ptr(), d.logits, d.bias, d.w13, d.sf13, d.w2, d.sf2, d.out,
                         d.workspace, d.ws_bytes, check=False)
    assert rc == moe.MOE_ERR_INVALID_ARG
    rc = moe.moe_forward(d.shape, d.x, d.logits, d.bias, d.w13, d.sf13, d.w2, d.sf2, d.x, d.workspace,
                         d.ws_bytes, check=False)
    assert rc == moe.MOE_ERR_INVALID_ARG                      # out aliases x
    torch.cuda.synchronize()
    pb.run_and_check()                                        # nothing launched by the rejected calls


def test_pack_mxfp4_scales_matches_the_layout():
    from checks import pack_mx_scales
    rng = np.random.default_rng(5)
    for batch, rows, K in ((1, 128, 128), (3, 256, 768), (2, 384, 6144)):
        src = rng.integers(0, 255, size=(batch, rows, K // 32), dtype=np.uint8)
        g = torch.from_numpy(src).cuda()
        out = torch.empty_like(g)
        moe.moe_pack_mxfp4_scales(g, batch, rows, K, out)
        torch.cuda.synchronize()
        assert np.array_equal(out.cpu().numpy(), pack_mx_scales(src))


def _routed_call(pb, ids, w):
    d = pb.dev
    ids_d = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).cuda()
    w_d = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda()
    d.out.zero_()
    rc = moe.moe_forward_routed(d.shape, d.x, ids_d, w_d, d.w13, d.sf13, d.w2, d.sf2, d.out, d.workspace,
                                d.ws_bytes, check=False)
    assert rc == moe.MOE_OK, moe.moe_last_error()
    torch.cuda.synchronize()
    return d.status()


# one shape per path: M <= 16 runs the single kernel, M = 40 the grouped kernels
ROUTED = [Workload("routed_small", 6, 512, 16, 3, 256, 1, 2.5, "normal", False),
          Workload("routed_grouped", 40, 512, 16, 3, 256, 1, 2.5, "normal", False)]


@pytest.mark.parametrize("wl", ROUTED, ids=lambda w: w.name)
def test_routed_entry_reproduces_the_internal_routing(wl):
    """Given the selection moe_forward computed, moe_forward_routed gives the same bytes."""
    pb = Problem(wl, seed=13)
    want, taps = pb.run_and_check()
    rc, st = _routed_call(pb, taps["topk_ids"], taps["topk_w"])
    assert rc == moe.MOE_OK and st == 0
    assert np.array_equal(pb.dev.out_bits(), want)


@pytest.mark.parametrize("wl", ROUTED, ids=lambda w: w.name)
def test_routed_entry_with_repeated_experts_matches_the_oracle(wl):
    """Caller selections may repeat an expert within a token; each occurrence counts."""
    pb = Problem(wl, seed=17)
    rng = np.random.default_rng(17)
    ids = rng.integers(0, wl.E, size=(wl.M, wl.topk)).astype(np.int32)
    ids[0, :] = ids[0, 0]                       # token 0 names one expert topk times
    ids[1, 1] = ids[1, 0]
    w = rng.uniform(0.05, 1.0, size=(wl.M, wl.topk)).astype(np.float32)
    rc, st = _routed_call(pb, ids, w)
    assert rc == moe.MOE_OK and st == 0
    res = oracle.forward_tokens(wl.shape(), pb.inputs.x, ids, w, *pb.ow)
    ok, worst = out_within_tol(pb.dev.out_bits(), res["ref"])
    assert ok, f"out outside tolerance (worst {worst:.3f} of the bound)"
    taps = pb.dev.taps()
    assert np.array_equal(taps["topk_ids"], ids)


@pytest.mark.parametrize("wl", ROUTED, ids=lambda w: w.name)
def test_routed_entry_reports_an_out_of_range_expert(wl):
    pb = Problem(wl, seed=19)
    ids = np.tile(np.arange(wl.topk, dtype=np.int32), (wl.M, 1))
    ids[wl.M - 1, 0] = wl.E                     # one ID past the last expert
    w = np.full((wl.M, wl.topk), 0.5, np.float32)
    rc, st = _routed_call(pb, ids, w)
    assert rc == moe.MOE_ERR_INVALID_ARG and st != 0
    pb.run_and_check()                          # the workspace serves the next call


# The pages' layer: 256 routed experts plus the shared expert fused as #256,
# top-9 ("[HIP] IQ2R: GLM-5.3 packed MoE path for TP4/TP8 on gfx950",
# Summary).  Here that is E = 257 expert weight sets, slots 0..7 the routed
# top-8 of the 256 routed experts, slot 8 expert 256 with weight 1, given to
# moe_forward_routed -- on the single kernel (M = 4) and the grouped kernels
# (M = 40), both weight formats.
SHARED = [Workload("shared_single", 4, 512, 257, 9, 256, 1, 2.5, "normal", False),
          Workload("shared_grouped", 40, 512, 257, 9, 256, 1, 2.5, "normal", False),
          Workload("shared_grouped_fp8", 40, 384, 257, 9, 256, 2, 2.5, "normal", False)]


@pytest.mark.parametrize("wl", SHARED, ids=lambda w: w.name)
def test_shared_expert_as_an_extra_slot(wl):
    pb = Problem(wl, seed=53)
    k = wl.topk - 1
    rng = np.random.default_rng(53)
    logits = rng.standard_normal((wl.M, wl.E - 1)).astype(np.float32)
    rid, rw = oracle.route(logits, None, k, wl.routed_scale)      # routed top-8 of the 256 routed experts
    ids = np.concatenate([rid, np.full((wl.M, 1), wl.E - 1, np.int32)], 1)
    w = np.concatenate([rw, np.ones((wl.M, 1), np.float32)], 1)
    rc, st = _routed_call(pb, ids, w)
    assert rc == moe.MOE_OK and st == 0
    taps = pb.dev.taps()
    assert np.array_equal(taps["topk_ids"], ids)
    assert np.all(taps["counts"][wl.E - 1] == wl.M)                   # every token uses the shared expert
    verify_call(wl, taps, pb.dev.out_bits(), None, None, pb.inputs.x, pb.ow, routed=(ids, w))
