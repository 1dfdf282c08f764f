"""Pin of the oracle's block-FP8 activation quantizer (CPU only).

For block-FP8 expert weights the tokens are quantized to E4M3 with one
power-of-two fp32 scale per 128 values along H (the group-128 FP8 activations
of "feat(glm52 mono): serve a BF16-attention checkpoint"; the scale value is
the reading that also fixes the mid scale: the smallest power of two 2^k,
k in [-126, 127], with amax <= 448 * 2^k, and 1 for an all-zero block).

The restatement below shares nothing with the oracle: the scale comes from a
linear search over k, the codes from a nearest-value search over the E4M3
magnitudes written out from the OCP OFP8 closed form (bias 7, 3 mantissa
bits, max 448, no infinities), ties to the even code, sign kept.  Codes and
scales are compared bit for bit on random rows and on crafted blocks whose
amax sits exactly on, just above and just below a binade edge 448 * 2^k, on
zero and subnormal blocks, and on blocks with a huge dynamic range.
"""
import bisect
import math

import numpy as np
import pytest

import oracle
from prefill_moe_route_b200.synth import W_FP8_BLOCK128, bf16_bits_to_f32, to_bf16_bits


def _e4m3_magnitudes():
    """(value, code) of every finite non-negative E4M3 code, from the closed form."""
    out = []
    for code in range(0x7F):                    # 0x7F is NaN
        e, m = code >> 3, code & 7
        val = m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out.append((val, code))
    return sorted(out)


_MAG = _e4m3_magnitudes()
_VALS = [v for v, _ in _MAG]


def e4m3_rne(u: float) -> int:
    """Nearest E4M3 code of an exact real u (|u| <= 448 here), ties to the even code."""
    a = abs(u)
    i = bisect.bisect_left(_VALS, a)
    cands = [j for j in (i - 1, i) if 0 <= j < len(_VALS)]
    best = min(cands, key=lambda j: (abs(_VALS[j] - a), _MAG[j][1] & 1))
    code = _MAG[best][1]
    return code | (0x80 if math.copysign(1.0, u) < 0 else 0)


def pow2_scale_search(amax: float) -> float:
    if amax == 0.0:
        return 1.0
    for k in range(-126, 128):
        if amax <= 448.0 * 2.0 ** k:
            return 2.0 ** k
    return 2.0 ** 127


def restated_quant_fp8_act(x_bits: np.ndarray):
    """x bf16 bits [M, H] -> (E4M3 codes [M, H], fp32 scales [M, H/128])."""
    xf = bf16_bits_to_f32(x_bits).astype(np.float64)
    M, H = xf.shape
    q = np.zeros((M, H), np.uint8)
    s = np.zeros((M, H // 128), np.float32)
    for t in range(M):
        for b in range(H // 128):
            blk = xf[t, b * 128:(b + 1) * 128]
            sc = pow2_scale_search(float(np.max(np.abs(blk))))
            s[t, b] = sc
            q[t, b * 128:(b + 1) * 128] = [e4m3_rne(float(v) / sc) for v in blk]   # exact in fp64
    return q, s


def _crafted_rows(rng):
    rows = []
    base = rng.standard_normal(128)
    for k in (-20, -3, 0, 1, 7, 40):
        edge = 448.0 * 2.0 ** k
        for amax in (edge, np.nextafter(np.float32(edge), np.float32(np.inf)),
                     np.nextafter(np.float32(edge), np.float32(0))):
            blk = base / np.max(np.abs(base)) * 0.9 * float(amax)
            blk[17] = -float(amax) if k % 2 else float(amax)          # the extreme, either sign
            rows.append(blk)
    rows.append(np.zeros(128))                                        # all-zero block: scale 1
    sub = np.zeros(128)
    sub[3], sub[90] = 2.0 ** -130, -(2.0 ** -133)                     # bf16 subnormals only
    rows.append(sub)
    wide = rng.standard_normal(128) * 1e-30
    wide[5] = 3.0e30                                                  # values far below the block's grid
    rows.append(wide)
    neg = -np.abs(rng.standard_normal(128)) * 1e-3                    # tiny negatives round to -0 or up
    rows.append(neg)
    return rows


def test_fp8_activation_quantizer_matches_the_restatement_on_crafted_blocks():
    rng = np.random.default_rng(41)
    rows = _crafted_rows(rng)
    H = 128 * len(rows)
    x = to_bf16_bits(np.concatenate(rows).astype(np.float32)[None, :])
    q, s = oracle.quant_act(W_FP8_BLOCK128, x)
    rq, rs = restated_quant_fp8_act(x)
    assert np.array_equal(s.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(q, rq)
    # the crafted edges take the intended binades (after the bf16 rounding of the inputs)
    xf = bf16_bits_to_f32(x)[0]
    for b in range(H // 128):
        amax = float(np.max(np.abs(xf[b * 128:(b + 1) * 128])))
        if amax > 0:
            assert amax <= 448.0 * float(s[0, b]) and (float(s[0, b]) == 2.0 ** -126 or amax > 224.0 * float(s[0, b]))


@pytest.mark.parametrize("M,H,scale", [(3, 512, 1.0), (2, 1536, 300.0), (4, 256, 1e-6)])
def test_fp8_activation_quantizer_matches_the_restatement_on_random_rows(M, H, scale):
    rng = np.random.default_rng(M * 1000 + H)
    x = to_bf16_bits((rng.standard_normal((M, H)) * scale).astype(np.float32))
    q, s = oracle.quant_act(W_FP8_BLOCK128, x)
    rq, rs = restated_quant_fp8_act(x)
    assert np.array_equal(s.view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(q, rq)


def test_restatement_catches_a_plausible_mistake():
    """A quantizer that took the scale of the wrong 128-block, or divided in a
    way that rounds, must disagree with the restatement."""
    rng = np.random.default_rng(5)
    x = to_bf16_bits((rng.standard_normal((1, 384)) * np.repeat([1.0, 50.0, 0.01], 128)).astype(np.float32))
    rq, rs = restated_quant_fp8_act(x)
    assert not np.array_equal(rs[0], np.roll(rs[0], 1))
    xf = bf16_bits_to_f32(x).astype(np.float64)[0]
    shifted = [e4m3_rne(float(v) / float(rs[0, (i // 128 + 1) % 3])) for i, v in enumerate(xf)]
    assert not np.array_equal(np.array(shifted, np.uint8), rq[0])


# ---------------------------------------------------------------- MXFP4 rows
_E2M1_MAG = [(0.0, 0), (0.5, 1), (1.0, 2), (1.5, 3), (2.0, 4), (3.0, 5), (4.0, 6), (6.0, 7)]   # OCP MX v1.0 E2M1


def e2m1_rne_sat(u: float) -> int:
    a = min(abs(u), 6.0)
    best = min(_E2M1_MAG, key=lambda vc: (abs(vc[0] - a), vc[1] & 1))[1]
    return best | (8 if math.copysign(1.0, u) < 0 else 0)


def restated_quant_mxfp4_act(x_bits: np.ndarray):
    """x bf16 bits [M, H] -> (packed E2M1 [M, H/2], E8M0 codes [M, H/32]): OCP MX v1.0 conversion,
    shared exponent floor(log2 amax) - 2 (clamped to [-127, 127]; 0 for an all-zero block)."""
    xf = bf16_bits_to_f32(x_bits).astype(np.float64)
    M, H = xf.shape
    q = np.zeros((M, H // 2), np.uint8)
    s = np.zeros((M, H // 32), np.uint8)
    for t in range(M):
        for b in range(H // 32):
            blk = xf[t, b * 32:(b + 1) * 32]
            amax = float(np.max(np.abs(blk)))
            e = -127 if amax == 0.0 else max(-127, min(127, math.floor(math.log2(amax)) - 2))
            s[t, b] = e + 127
            codes = [e2m1_rne_sat(float(v) / 2.0 ** e) for v in blk]
            for i in range(16):
                q[t, b * 16 + i] = codes[2 * i] | (codes[2 * i + 1] << 4)
    return q, s


@pytest.mark.parametrize("M,H,scale", [(2, 512, 1.0), (3, 256, 1e-3), (1, 1024, 1e4)])
def test_mxfp4_activation_quantizer_matches_the_restatement(M, H, scale):
    from prefill_moe_route_b200.synth import W_MXFP4
    rng = np.random.default_rng(M + H)
    v = (rng.standard_normal((M, H)) * scale).astype(np.float32)
    v[0, :32] = 0.0                                    # an all-zero block
    v[0, 32:64] = np.float32(6.0 * 2.0 ** 3)           # amax exactly 6 * 2^k: elements land on 6
    x = to_bf16_bits(v)
    q, s = oracle.quant_act(W_MXFP4, x)
    rq, rs = restated_quant_mxfp4_act(x)
    assert np.array_equal(s, rs)
    assert np.array_equal(q, rq)
