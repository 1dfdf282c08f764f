"""The pages' layer is top-9: the routed top-8 plus a shared expert, numbered
after the routed ones, that every token uses ("[HIP] IQ2R: GLM-5.3 packed MoE
path for TP4/TP8 on gfx950", Summary: 256 routed experts, the shared one fused
as #256).  Here
that is an extra slot of the same call: E + 1 experts in the weight tensors,
the routed selection in slots 0..k-1 and expert E with its own weight in slot
k, given to moe_forward_routed.  These CPU tests pin that reading on the
oracle: the extra slot adds exactly the shared expert's own output (the
combine is a sum over slots in order), and nothing else changes."""
import numpy as np
import pytest

import oracle
from prefill_moe_route_b200.synth import W_FP8_BLOCK128, W_MXFP4, to_bf16_bits


def _quant(wfmt, f13, f2):
    if wfmt == W_MXFP4:
        return (*oracle.quant_mxfp4(f13), *oracle.quant_mxfp4(f2))
    return (*oracle.quant_fp8_block128(f13), *oracle.quant_fp8_block128(f2))


@pytest.mark.parametrize("wfmt", [W_MXFP4, W_FP8_BLOCK128])
def test_shared_expert_slot_adds_its_own_output(wfmt):
    rng = np.random.default_rng(31 + wfmt)
    M, H, I, E, k = 3, 256, 128, 6, 2          # E routed experts + 1 shared (index E)
    x = to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids, tw = oracle.route(logits, None, k, 2.5)
    f13 = (rng.standard_normal((E + 1, 2 * I, H)) * 0.02).astype(np.float32)
    f2 = (rng.standard_normal((E + 1, H, I)) * 0.02).astype(np.float32)
    w = _quant(wfmt, f13, f2)

    def call(topk, sel, wts):
        shape = dict(M=M, H=H, I=I, E=E + 1, topk=topk, routed_scale=2.5, wfmt=wfmt)
        return oracle.forward_tokens(shape, x, sel, wts, *w)

    w_shared = np.float32(1.0)
    routed = call(k, ids, tw)
    shared = call(1, np.full((M, 1), E, np.int32), np.full((M, 1), w_shared, np.float32))
    both = call(k + 1, np.concatenate([ids, np.full((M, 1), E, np.int32)], 1),
                np.concatenate([tw, np.full((M, 1), w_shared, np.float32)], 1))
    # same operations in the same order: exact in fp64
    assert np.array_equal(both["ref"], routed["ref"] + shared["ref"])
    # the routed slots' mid blocks are untouched by the extra slot
    rows = (np.arange(M)[:, None] * (k + 1) + np.arange(k)[None, :]).reshape(-1)
    assert np.array_equal(both["midq"][rows], routed["midq"])
    assert np.array_equal(both["midqs"][rows], routed["midqs"])
    # and the shared slot's mid is the shared expert's alone
    assert np.array_equal(both["midq"][np.arange(M) * (k + 1) + k], shared["midq"])
