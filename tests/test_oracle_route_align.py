"""Pins of the oracle's routing and pair sort (CPU only): brute force with
numpy's lexsort / stable argsort, invariants, crafted ties."""
import numpy as np
import pytest

import oracle


def _sel(logits, bias):
    s = np.vectorize(oracle.sigmoid_spec, otypes=[np.float32])(logits.astype(np.float32))
    sel = s + (bias.astype(np.float32) if bias is not None else np.float32(0))
    return s.astype(np.float32), sel.astype(np.float32)


@pytest.mark.parametrize("M,E,k,use_bias", [(7, 8, 2, True), (5, 64, 8, False), (3, 256, 8, True), (4, 9, 9, True)])
def test_route_brute_force(M, E, k, use_bias):
    rng = np.random.default_rng(M * 1000 + E)
    logits = rng.standard_normal((M, E)).astype(np.float32)
    bias = (rng.standard_normal(E) * 0.1).astype(np.float32) if use_bias else None
    ids, w = oracle.route(logits, bias, k, 2.5)
    s, sel = _sel(logits, bias)
    for t in range(M):
        order = np.lexsort((np.arange(E), -sel[t].astype(np.float64)))   # by (-sel, id)
        assert list(ids[t]) == list(order[:k])
        assert len(set(ids[t])) == k
        # weights: normalized selected sigmoids times the routed scale
        tot = float(np.sum(w[t].astype(np.float64))) / 2.5
        assert abs(tot - 1.0) <= k * 2.0 ** -23
        ratios = w[t].astype(np.float64) / s[t][ids[t]].astype(np.float64)
        assert np.allclose(ratios, ratios[0], rtol=4e-7)


def test_route_ties_go_to_lower_id():
    logits = np.zeros((2, 16), np.float32)        # all sigmoids equal
    ids, w = oracle.route(logits, None, 4, 1.0)
    assert ids.tolist() == [[0, 1, 2, 3]] * 2
    assert np.all(w == np.float32(0.25))
    logits2 = np.full((1, 8), -1.0, np.float32)
    logits2[0, [6, 3]] = 0.5                      # tie between 3 and 6 at the top
    ids2, _ = oracle.route(logits2, None, 3, 1.0)
    assert ids2.tolist() == [[3, 6, 0]]


def test_route_bias_changes_selection_not_weights():
    logits = np.array([[0.0, 0.1, 0.2, 0.3]], np.float32)
    bias = np.array([1.0, 0.0, 0.0, 0.0], np.float32)
    ids, w = oracle.route(logits, bias, 2, 1.0)
    assert ids.tolist() == [[0, 3]]
    s0, s3 = oracle.sigmoid_spec(0.0), oracle.sigmoid_spec(0.3)
    assert abs(w[0, 0] - s0 / (s0 + s3)) < 1e-7 and abs(w[0, 1] - s3 / (s0 + s3)) < 1e-7


@pytest.mark.parametrize("M,E,k", [(1, 4, 1), (33, 8, 2), (100, 256, 8), (17, 5, 5)])
def test_align_matches_stable_argsort(M, E, k):
    rng = np.random.default_rng(M + E)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(M)]).astype(np.int32)
    counts, offsets, sp, inv = oracle.align(ids, E)
    flat = ids.reshape(-1)
    ref = np.argsort(flat, kind="stable")
    assert np.array_equal(sp, ref)
    assert np.array_equal(counts, np.bincount(flat, minlength=E))
    assert offsets[0] == 0 and offsets[-1] == M * k and np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(inv[sp], np.arange(M * k))
    # every token appears exactly k times; inside an expert, tokens ascend
    assert np.array_equal(np.bincount(sp // k, minlength=M), np.full(M, k))
    for e in range(E):
        seg = sp[offsets[e]:offsets[e + 1]]
        assert np.all(flat[seg] == e) and np.all(np.diff(seg) > 0)
