"""Negative controls of the parity checker (CPU only).

The checker the GPU parity tests use (checks.verify_call) is given a candidate
built from the oracle itself -- which it must accept -- and then copies of that
candidate with one planted mistake each, which it must reject: a flipped
nibble of a mid code, the permutation rolled by one, a corrupted mid scale, a
corrupted expert-weight scale upstream of the whole call, and output rows
shifted by one token.  Mistakes are planted on the CPU, in oracle results.
"""
import numpy as np
import pytest

import oracle
from checks import verify_call
from prefill_moe_route_b200.synth import W_FP8_BLOCK128, W_MXFP4, Inputs, Workload

WLS = [Workload("ctl_mx", 6, 256, 8, 2, 256, W_MXFP4, 2.5, "normal", True),
       Workload("ctl_fp8", 5, 256, 8, 3, 256, W_FP8_BLOCK128, 2.5, "normal", True)]


def _weights(wl, inputs):
    q = [[], [], [], []]
    for e in range(wl.E):
        if wl.wfmt == W_MXFP4:
            parts = (*oracle.quant_mxfp4(inputs.w13(e)), *oracle.quant_mxfp4(inputs.w2(e)))
        else:
            parts = (*oracle.quant_fp8_block128(inputs.w13(e)), *oracle.quant_fp8_block128(inputs.w2(e)))
        for lst, v in zip(q, parts):
            lst.append(v)
    return [np.stack(v) for v in q]


def _candidate(wl, inputs, ow):
    """What a correct implementation leaves behind: taps in sorted order and bf16 out."""
    ids, tw = oracle.route(inputs.logits, inputs.bias, wl.topk, wl.routed_scale)
    counts, offsets, sp, inv = oracle.align(ids, wl.E)
    res = oracle.forward_tokens(wl.shape(), inputs.x, ids, tw, *ow)
    taps = {"topk_ids": ids, "topk_w": tw, "counts": counts, "offsets": offsets, "sorted_pairs": sp, "inv": inv,
            "midq": res["midq"][sp].copy(), "midqs": res["midqs"][sp].copy()}
    return taps, res["out"].copy()


@pytest.fixture(params=WLS, ids=lambda w: w.name)
def problem(request):
    wl = request.param
    inputs = Inputs(wl, seed=9)
    ow = _weights(wl, inputs)
    taps, out = _candidate(wl, inputs, ow)
    return wl, inputs, ow, taps, out


def _verify(wl, inputs, ow, taps, out):
    return verify_call(wl, taps, out, inputs.logits, inputs.bias, inputs.x, ow)


def test_checker_accepts_the_oracle_itself(problem):
    _verify(*problem)


def test_flipped_mid_nibble_is_rejected(problem):
    wl, inputs, ow, taps, out = problem
    t = dict(taps, midq=taps["midq"].copy())
    t["midq"][1, 5] ^= 0x40                     # an exponent bit: far more than one E4M3 step
    with pytest.raises(AssertionError, match="mid codes"):
        _verify(wl, inputs, ow, t, out)


def test_rolled_permutation_is_rejected(problem):
    wl, inputs, ow, taps, out = problem
    t = dict(taps, sorted_pairs=np.roll(taps["sorted_pairs"], 1))
    with pytest.raises(AssertionError, match="sorted pairs"):
        _verify(wl, inputs, ow, t, out)


def test_corrupted_mid_scale_is_rejected(problem):
    wl, inputs, ow, taps, out = problem
    t = dict(taps, midqs=taps["midqs"].copy())
    t["midqs"][0, 0] *= 4.0                     # two binades off
    with pytest.raises(AssertionError, match="mid codes"):
        _verify(wl, inputs, ow, t, out)
    t = dict(taps, midqs=taps["midqs"] * 2.0)   # one binade off everywhere: more than the 1 % allowance
    with pytest.raises(AssertionError, match="binade"):
        _verify(wl, inputs, ow, t, out)


def test_corrupted_weight_scale_is_rejected(problem):
    """A candidate computed with one expert's weight scales corrupted (the
    first selected expert of token 0, every block x16) fails the mid check."""
    wl, inputs, ow, taps, out = problem
    bad = [a.copy() for a in ow]
    e = int(taps["topk_ids"][0, 0])
    if wl.wfmt == W_MXFP4:
        bad[1][e] = np.minimum(bad[1][e].astype(np.int32) + 4, 254).astype(np.uint8)
    else:
        bad[1][e] *= 16.0
    t, o = _candidate(wl, inputs, bad)
    with pytest.raises(AssertionError):
        _verify(wl, inputs, ow, t, o)


def test_output_rows_shifted_by_one_token_are_rejected(problem):
    wl, inputs, ow, taps, out = problem
    with pytest.raises(AssertionError, match="out outside tolerance"):
        _verify(wl, inputs, ow, taps, np.roll(out, 1, axis=0))
