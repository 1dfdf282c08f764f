"""Pins of the oracle's codecs (CPU only).

Each check ties the oracle to something outside itself: literal values of the
OCP MX v1.0 / OCP OFP8 specifications (tests/golden/), torch's own fp8 and
bf16 conversions, brute-force nearest-value search, hand-computed cases.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import read_golden


def _golden(name):
    out = {}
    for code, val in read_golden(name):
        out[int(code, 16)] = float(val)
    return out


def test_e2m1_decode_matches_ocp_table():
    table = _golden("ocp_e2m1_values.txt")
    assert len(table) == 16
    for code, val in table.items():
        got = oracle.e2m1_value(code)
        assert got == val and math.copysign(1, got) == math.copysign(1, val), hex(code)


def test_e4m3_decode_matches_ocp_points_and_torch():
    for code, val in _golden("ocp_e4m3_points.txt").items():
        got = oracle.e4m3_value(code)
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val, hex(code)
    # every code against torch's float8_e4m3fn decode (a library routine)
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        got = oracle.e4m3_value(c)
        if math.isnan(ref[c]):
            assert math.isnan(got), hex(c)
        else:
            assert got == float(ref[c]), hex(c)


def test_e8m0_decode():
    assert oracle.e8m0_value(127) == 1.0
    assert oracle.e8m0_value(0) == 2.0 ** -127
    assert oracle.e8m0_value(254) == 2.0 ** 127
    assert oracle.e8m0_value(130) == 8.0
    assert math.isnan(oracle.e8m0_value(255))


def _nearest_even(v, codes_vals):
    """Brute force: nearest representable magnitude, ties to the even code."""
    best = None
    for code, val in codes_vals:
        d = abs(abs(v) - val)
        if best is None or d < best[0] or (d == best[0] and code % 2 == 0 and best[1] % 2 == 1):
            best = (d, code)
    return best[1]


def test_e2m1_encode_brute_force():
    table = _golden("ocp_e2m1_values.txt")
    pos = sorted((c, v) for c, v in table.items() if c < 8)
    mags = [v for _, v in pos]
    rng = np.random.default_rng(1)
    vals = list(rng.uniform(-8, 8, 4000)) + list(rng.uniform(-1, 1, 1000))
    mids = [(a + b) / 2 for a, b in zip(mags, mags[1:])]
    vals += mids + [-m for m in mids] + [6.0, 6.5, 7.0, 100.0, -100.0, 0.25, 0.74, 0.76]
    for v in vals:
        code = oracle.e2m1_encode(float(v))
        expect = _nearest_even(v, pos)
        assert code & 7 == expect, (v, code, expect)
        assert (code >> 3) == (1 if math.copysign(1, v) < 0 else 0), v


def test_e4m3_encode_brute_force_and_torch():
    pos = [(c, oracle.e4m3_value(c)) for c in range(0x7F)]  # decode pinned above
    rng = np.random.default_rng(2)
    vals = list(rng.uniform(-500, 500, 2000)) + list(rng.normal(0, 1, 2000)) + list(rng.normal(0, 0.01, 1000))
    mags = [v for _, v in pos]
    mids = [(a + b) / 2 for a, b in zip(mags, mags[1:])]
    vals += mids + [-m for m in mids] + [448.0, 449.0, 464.0, 470.0, 1e6, -1e6]
    for v in vals:
        code = oracle.e4m3_encode(float(v))
        assert code & 0x7F == _nearest_even(v, pos), (v, code)
    # torch's round-to-nearest-even conversion agrees inside the finite range
    inr = np.array([v for v in vals if abs(v) <= 448.0], np.float32)
    tc = torch.from_numpy(inr).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    mine = np.array([oracle.e4m3_encode(float(v)) for v in inr], np.uint8)
    nz = inr != 0
    assert np.array_equal(tc[nz], mine[nz])


def test_bf16_encode_matches_torch():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.normal(0, 1, 5000), rng.normal(0, 1e-30, 100), [1.0, -2.5, 3.00390625]]).astype(np.float32)
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    mine = np.array([oracle.bf16_encode(float(x)) for x in v], np.uint16)
    assert np.array_equal(ref, mine)


@pytest.mark.parametrize("amax,code", [
    (1.0, 125),            # floor(log2 1) = 0 -> 2^-2
    (48.0, 130),           # 48 = 6 * 2^3: floor(log2) = 5 -> 2^3, elements exactly 6
    (7.99, 127),           # floor(log2) = 2 -> 2^0: 7.99 saturates to 6
    (0.0, 0),
    (2.0 ** -130, 0),      # exponent clamped to -127
    (0.75, 124),           # floor(log2 0.75) = -1 -> 2^-3
])
def test_mx_scale_rule_crafted(amax, code):
    assert oracle.mx_scale_code(amax) == code


def test_mx_block_quant_crafted():
    blk = np.zeros(32, np.float32)
    blk[:8] = [6.0, -6.0, 3.0, 1.5, 0.5, 0.0, 4.0, 2.0]
    blk *= 2.0 ** 3                                  # amax = 48 -> X = 8
    q, s = oracle.quant_mxfp4(blk[None, :])
    assert s[0, 0] == 130
    codes = [(q[0, i // 2] >> (4 * (i % 2))) & 15 for i in range(8)]
    assert codes == [0x7, 0xF, 0x5, 0x3, 0x1, 0x0, 0x6, 0x4]
    blk2 = np.full(32, 7.99, np.float32)
    q2, s2 = oracle.quant_mxfp4(blk2[None, :])
    assert s2[0, 0] == 127 and q2[0, 0] == 0x77      # saturated to 6


def test_pow2_scale_brute_force():
    rng = np.random.default_rng(4)
    vals = np.concatenate([np.exp(rng.uniform(-60, 60, 3000)), 448.0 * 2.0 ** np.arange(-20, 20),
                           448.0 * 2.0 ** np.arange(-20, 20) * (1 + 2 ** -20)]).astype(np.float32)
    for a in vals:
        a = float(a)
        k = -126
        while a > 448.0 * 2.0 ** k:
            k += 1
        assert oracle.pow2_scale_e4m3(a) == 2.0 ** k, a
    assert oracle.pow2_scale_e4m3(0.0) == 1.0


def test_fp8_block_quant_matches_definition():
    rng = np.random.default_rng(5)
    w = (rng.standard_normal((256, 384)) * 0.02).astype(np.float32)
    w[128:, 256:] = 0.0                              # an all-zero block -> scale 1
    q, s = oracle.quant_fp8_block128(w)
    assert s.shape == (2, 3)
    assert s[1, 2] == 1.0 and np.all(q[128:, 256:] == 0)
    blk = w[:128, 128:256]
    amax = np.float32(np.abs(blk).max())
    assert s[0, 1] == np.float32(amax / np.float32(448.0))
    # dequantized block reproduces the input within half an E4M3 step
    deq = torch.from_numpy(q[:128, 128:256].copy()).view(torch.float8_e4m3fn).float().numpy() * s[0, 1]
    assert np.all(np.abs(deq - blk) <= np.abs(blk) * 2.0 ** -4 + s[0, 1] * 2.0 ** -10)


def test_exp_and_sigmoid_spec_against_libm():
    xs = np.concatenate([np.linspace(-87, 88, 200001), np.linspace(-1, 1, 20001)]).astype(np.float32)
    worst = 0
    for x in xs[::7]:
        got = oracle.exp_spec(float(x))
        ref = np.float32(math.exp(float(x)))
        ulp = np.spacing(np.float32(ref))
        worst = max(worst, abs(got - float(ref)) / float(ulp))
    assert worst <= 2.0, worst
    assert oracle.exp_spec(0.0) == 1.0
    assert oracle.sigmoid_spec(0.0) == 0.5
    for l in (-20.0, -3.0, -0.5, 0.7, 4.0, 15.0):
        assert abs(oracle.sigmoid_spec(l) - 1 / (1 + math.exp(-l))) <= 3e-7
