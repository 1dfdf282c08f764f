"""Test-side helpers: independent dequantization (lookup tables from the OCP
specs and torch's fp8 decode) and the parity comparisons used by the tests."""
import numpy as np
import torch

from conftest import read_golden

_E2M1 = np.zeros(16, np.float64)
for _code, _val in read_golden("ocp_e2m1_values.txt"):
    _E2M1[int(_code, 16)] = float(_val)


def e4m3_values(codes: np.ndarray) -> np.ndarray:
    c = np.ascontiguousarray(codes, np.uint8)
    return torch.from_numpy(c.copy()).view(torch.float8_e4m3fn).double().numpy()


def unpack_e2m1(q: np.ndarray) -> np.ndarray:
    q = np.asarray(q, np.uint8)
    out = np.empty(q.shape[:-1] + (q.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = q & 15
    out[..., 1::2] = q >> 4
    return out


def deq_mxfp4(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    vals = _E2M1[unpack_e2m1(q)]
    scale = np.repeat(2.0 ** (np.asarray(s, np.float64) - 127.0), 32, axis=-1)
    return vals * scale


def deq_fp8_block(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    vals = e4m3_values(q)
    sc = np.repeat(np.repeat(np.asarray(s, np.float64), 128, axis=-2), 128, axis=-1)
    return vals * sc


def e4m3_ordinal(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, np.int32)
    mag = c & 0x7F
    return np.where(c & 0x80, -mag, mag)


def compare_mid(q_gpu, s_gpu, q_ref, s_ref):
    """midq within one E4M3 step, midqs exact; a block whose scale differs by
    exactly one binade (amax on a binade edge) is counted, not compared.
    q_*: [rows, I] codes, s_*: [rows, I/128].  Returns (bad_codes, binade_edges)."""
    rows, I = q_ref.shape
    nb = I // 128
    bad = 0
    edges = 0
    for b in range(nb):
        same = s_gpu[:, b] == s_ref[:, b]
        ratio = s_gpu[:, b].astype(np.float64) / s_ref[:, b].astype(np.float64)
        edge = ~same & ((ratio == 2.0) | (ratio == 0.5))
        other = ~same & ~edge
        bad += int(other.sum()) * 128
        edges += int(edge.sum())
        d = np.abs(e4m3_ordinal(q_gpu[same, b * 128:(b + 1) * 128]) - e4m3_ordinal(q_ref[same, b * 128:(b + 1) * 128]))
        bad += int((d > 1).sum())
    return bad, edges


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def out_within_tol(out_bits, ref, atol=2e-2, rtol=2e-2):
    o = bf16_to_f64(out_bits)
    err = np.abs(o - ref)
    lim = atol + rtol * np.abs(ref)
    return bool(np.all(err <= lim)), float(np.max(err / lim)) if err.size else 0.0


def pack_mx_scales(s: np.ndarray) -> np.ndarray:
    """Row-major E8M0 scales [..., rows, K/32] -> the packed byte order of
    moe_pack_mxfp4_scales: [..., rows/128, K/128] blocks of 512 bytes, row r
    of a 128-row tile at byte 16 * (r % 32) + 4 * (r // 32), its 4 scales in
    column order (the tensor cores' 32x128-bit scale-factor tile)."""
    s = np.ascontiguousarray(s, np.uint8)
    lead, rows, k32 = s.shape[:-2], s.shape[-2], s.shape[-1]
    x = s.reshape(lead + (rows // 128, 4, 32, k32 // 4, 4))   # tile, (r % 128) // 32, r % 32, group, scale
    x = np.moveaxis(x, -2, -4)                                  # tile, group, (r % 128) // 32, r % 32, scale
    x = np.swapaxes(x, -3, -2)                                  # tile, group, r % 32, (r % 128) // 32, scale
    return np.ascontiguousarray(x).reshape(s.shape)


def verify_call(wl, taps, out_bits, logits, bias, x_bits, oracle_weights, tokens=None, routed=None):
    """The parity bar of one MoE call, raising AssertionError on any miss.

    taps: the workspace debug taps of the call (topk_ids, topk_w, counts,
    offsets, sorted_pairs, inv, midq, midqs); out_bits: bf16 out [M, H] (all
    tokens).  Routing and the sort are compared bit for bit in full; mid
    (each code within one E4M3 step, scales exact, binade-edge blocks at most
    1 %) and out (2e-2 + 2e-2 relative) on `tokens` (all when None).
    routed: (ids, w) of a caller's selection instead of routing the logits."""
    import oracle
    if routed is None:
        ids, tw = oracle.route(logits, bias, wl.topk, wl.routed_scale)
    else:
        ids, tw = routed
    if not np.array_equal(taps["topk_ids"], ids):
        raise AssertionError(f"routing ids differ ({near_tie_flips(taps['topk_ids'], ids, logits, bias)})")
    assert np.array_equal(np.asarray(taps["topk_w"], np.float32).view(np.uint32),
                          np.asarray(tw, np.float32).view(np.uint32)), "routing weights differ"
    counts, offsets, sp, inv = oracle.align(ids, wl.E)
    assert np.array_equal(taps["counts"], counts), "counts differ"
    assert np.array_equal(taps["offsets"], offsets), "offsets differ"
    assert np.array_equal(taps["sorted_pairs"], sp), "sorted pairs differ"
    assert np.array_equal(taps["inv"], inv), "inverse permutation differs"
    toks = np.arange(wl.M, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    res = oracle.forward_tokens(wl.shape(), x_bits, ids, tw, *oracle_weights, tokens=toks)
    rows = inv[(toks[:, None] * wl.topk + np.arange(wl.topk)[None, :]).reshape(-1)]
    bad, edges = compare_mid(taps["midq"][rows], taps["midqs"][rows], res["midq"], res["midqs"])
    nblocks = rows.size * (wl.I // 128)
    assert bad == 0, f"{bad} mid codes off by more than one E4M3 step"
    assert edges <= max(1, nblocks // 100), f"{edges} of {nblocks} mid scales differ by a binade"
    ok, worst = out_within_tol(np.asarray(out_bits)[toks], res["ref"])
    assert ok, f"out outside tolerance (worst {worst:.3f} of the bound)"
    return res, edges


def near_tie_flips(got_ids, ref_ids, logits, bias, ulps=2):
    """Diagnosis of a routing mismatch: how many mismatched tokens have, for
    every expert chosen on one side only, a selection score within `ulps` fp32
    ulps of the other side's weakest choice (a near-tie flip)."""
    import oracle
    bad = np.nonzero(np.any(np.asarray(got_ids) != np.asarray(ref_ids), axis=1))[0]
    near = 0
    for t in bad:
        sel = np.array([oracle.sigmoid_spec(float(v)) for v in logits[t]], np.float32)
        if bias is not None:
            sel = (sel + np.asarray(bias, np.float32)).astype(np.float32)
        a, b = set(np.asarray(got_ids)[t].tolist()), set(np.asarray(ref_ids)[t].tolist())
        diff = sorted(a ^ b)
        if not diff:
            continue        # same experts, another order
        lo = float(min(sel[list(b)]))
        if all(abs(float(sel[e]) - lo) <= ulps * float(np.spacing(np.float32(lo))) for e in diff):
            near += 1
    return f"{len(bad)} tokens differ, {near} of them near-tie flips within {ulps} ulp"
