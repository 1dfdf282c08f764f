"""Pins of the oracle's forward (CPU only): brute force on tiny shapes with
numpy matrix products over independently dequantized weights, and special
cases whose result is known in closed form."""
import numpy as np
import pytest
import torch

import oracle
from checks import compare_mid, deq_fp8_block, deq_mxfp4, e4m3_values
from test_oracle_act_quant import pow2_scale_search, restated_quant_fp8_act, restated_quant_mxfp4_act
from prefill_moe_route_b200.synth import W_FP8_BLOCK128, W_MXFP4, to_bf16_bits


def _weights(wfmt, E, H, I, rng, scale=0.02):
    f13 = (rng.standard_normal((E, 2 * I, H)) * scale).astype(np.float32)
    f2 = (rng.standard_normal((E, H, I)) * scale).astype(np.float32)
    return f13, f2


def _quant(wfmt, f13, f2):
    if wfmt == W_MXFP4:
        return (*oracle.quant_mxfp4(f13), *oracle.quant_mxfp4(f2))
    return (*oracle.quant_fp8_block128(f13), *oracle.quant_fp8_block128(f2))


def _deq(wfmt, q, s):
    return deq_mxfp4(q, s) if wfmt == W_MXFP4 else deq_fp8_block(q, s)


def brute_forward(shape, x_bits, ids, tw, w13, s13, w2, s2):
    """Dense numpy version of the MoE call on the oracle's quantized inputs."""
    wfmt, M, H, I, k = shape["wfmt"], shape["M"], shape["H"], shape["I"], shape["topk"]
    # the activation quantizers restated independently of the oracle
    if wfmt == W_MXFP4:
        xq, xs = restated_quant_mxfp4_act(x_bits)
        xd = deq_mxfp4(xq, xs)
    else:
        xq, xs = restated_quant_fp8_act(x_bits)
        xd = e4m3_values(xq) * np.repeat(xs.astype(np.float64), 128, -1)
    W13 = _deq(wfmt, w13, s13)
    W2 = _deq(wfmt, w2, s2)
    midq = np.zeros((M * k, I), np.uint8)
    midqs = np.zeros((M * k, I // 128), np.float32)
    ref = np.zeros((M, H))
    for t in range(M):
        for j in range(k):
            e = ids[t, j]
            g = W13[e] @ xd[t]
            gate = g[:I].astype(np.float32).astype(np.float64)
            up = g[I:].astype(np.float32).astype(np.float64)
            mid = (gate / (1.0 + np.exp(-gate)) * up).astype(np.float32)
            md = np.zeros(I)
            for b in range(I // 128):
                blk = mid[b * 128:(b + 1) * 128]
                s = np.float32(pow2_scale_search(float(np.abs(blk).max())))
                codes = torch.from_numpy((blk / s).astype(np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
                midq[t * k + j, b * 128:(b + 1) * 128] = codes
                midqs[t * k + j, b] = s
                md[b * 128:(b + 1) * 128] = e4m3_values(codes) * float(s)
            ref[t] += float(tw[t, j]) * (W2[e] @ md)
    return midq, midqs, ref


CASES = [
    dict(wfmt=W_MXFP4, M=3, H=256, I=128, E=4, topk=2),
    dict(wfmt=W_MXFP4, M=2, H=512, I=256, E=3, topk=3),
    dict(wfmt=W_FP8_BLOCK128, M=3, H=256, I=128, E=4, topk=2),
    dict(wfmt=W_FP8_BLOCK128, M=2, H=384, I=256, E=2, topk=1),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"fmt{c['wfmt']}-M{c['M']}-H{c['H']}-I{c['I']}")
def test_forward_brute_force(case):
    rng = np.random.default_rng(sum(case.values()))
    shape = dict(case, routed_scale=2.5)
    M, H, I, E, k = case["M"], case["H"], case["I"], case["E"], case["topk"]
    x = to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    logits = rng.standard_normal((M, E)).astype(np.float32)
    ids, tw = oracle.route(logits, None, k, 2.5)
    f13, f2 = _weights(case["wfmt"], E, H, I, rng)
    w13, s13, w2, s2 = _quant(case["wfmt"], f13, f2)
    res = oracle.forward_tokens(shape, x, ids, tw, w13, s13, w2, s2)
    bq, bs, bref = brute_forward(shape, x, ids, tw, w13, s13, w2, s2)
    bad, edges = compare_mid(res["midq"], res["midqs"], bq, bs)
    assert bad == 0 and edges == 0
    assert np.allclose(res["ref"], bref, rtol=1e-9, atol=1e-12)
    # bf16 output is the rounded fp64 result
    o = (res["out"].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert np.all(np.abs(o - bref) <= np.abs(bref) * 2.0 ** -8 + 1e-30)
    # a token subset gives the same rows
    sub = oracle.forward_tokens(shape, x, ids, tw, w13, s13, w2, s2, tokens=np.array([M - 1], np.int32))
    assert np.array_equal(sub["ref"][0], res["ref"][M - 1])
    assert np.array_equal(sub["midq"], res["midq"][(M - 1) * k:M * k])


def test_one_hot_weights_give_quantized_x():
    """Gate row n picks x[h1], up row n picks x[h2]: mid = silu(xq[h1]) * xq[h2]."""
    M, H, I, E, k = 2, 256, 128, 1, 1
    rng = np.random.default_rng(11)
    x = to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    f13 = np.zeros((E, 2 * I, H), np.float32)
    h1 = rng.integers(0, H, I)
    h2 = rng.integers(0, H, I)
    f13[0, np.arange(I), h1] = 1.0
    f13[0, I + np.arange(I), h2] = 1.0
    f2 = np.zeros((E, H, I), np.float32)
    w13, s13, w2, s2 = _quant(W_MXFP4, f13, f2)
    shape = dict(wfmt=W_MXFP4, M=M, H=H, I=I, E=E, topk=k, routed_scale=1.0)
    ids = np.zeros((M, 1), np.int32)
    tw = np.ones((M, 1), np.float32)
    res = oracle.forward_tokens(shape, x, ids, tw, w13, s13, w2, s2)
    xq, xs = oracle.quant_act(W_MXFP4, x)
    xd = deq_mxfp4(xq, xs)
    for t in range(M):
        g = xd[t, h1].astype(np.float32).astype(np.float64)
        u = xd[t, h2].astype(np.float32).astype(np.float64)
        mid = (g / (1 + np.exp(-g)) * u).astype(np.float32)
        s = oracle.pow2_scale_e4m3(float(np.abs(mid).max()))
        assert res["midqs"][t, 0] == s
        codes = torch.from_numpy(mid / np.float32(s)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        zero = lambda c: np.where(c == 0x80, 0, c)          # +0 and -0 encode the same value
        assert np.array_equal(zero(res["midq"][t]), zero(codes))
    assert np.all(res["ref"] == 0.0)            # zero down weights -> zero output


@pytest.mark.parametrize("wfmt", [W_MXFP4, W_FP8_BLOCK128])
def test_special_cases(wfmt):
    M, H, I, E, k = 3, 256, 128, 4, 2
    rng = np.random.default_rng(12)
    x = to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    logits = rng.standard_normal((M, E)).astype(np.float32)
    f13, f2 = _weights(wfmt, E, H, I, rng)
    w13, s13, w2, s2 = _quant(wfmt, f13, f2)
    shape = dict(wfmt=wfmt, M=M, H=H, I=I, E=E, topk=k, routed_scale=1.0)
    ids, tw = oracle.route(logits, None, k, 1.0)
    base = oracle.forward_tokens(shape, x, ids, tw, w13, s13, w2, s2)["ref"]
    # doubling the routed scale doubles the result exactly
    ids2, tw2 = oracle.route(logits, None, k, 2.0)
    assert np.array_equal(ids2, ids) and np.array_equal(tw2, tw * 2)
    dbl = oracle.forward_tokens(dict(shape, routed_scale=2.0), x, ids2, tw2, w13, s13, w2, s2)["ref"]
    assert np.array_equal(dbl, 2 * base)
    # x = 0 -> out = 0
    z = oracle.forward_tokens(shape, np.zeros_like(x), ids, tw, w13, s13, w2, s2)["ref"]
    assert np.all(z == 0.0)
    # the combine is the routing-weighted sum of single-expert (k = 1) results
    acc = np.zeros_like(base)
    for j in range(k):
        one = oracle.forward_tokens(dict(shape, topk=1), x, ids[:, j:j + 1].copy(),
                                    np.ones((M, 1), np.float32), w13, s13, w2, s2)["ref"]
        acc += tw[:, j:j + 1].astype(np.float64) * one
    assert np.allclose(acc, base, rtol=1e-12, atol=1e-15)
    # k = E: every expert contributes (dense weighted sum)
    idsE, twE = oracle.route(logits, None, E, 1.0)
    assert all(sorted(r) == list(range(E)) for r in idsE.tolist())
    _, _, bref = brute_forward(dict(shape, topk=E), x, idsE, twE, w13, s13, w2, s2)
    assert np.allclose(oracle.forward_tokens(dict(shape, topk=E), x, idsE, twE, w13, s13, w2, s2)["ref"],
                       bref, rtol=1e-9, atol=1e-12)
