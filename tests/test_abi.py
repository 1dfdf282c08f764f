"""The C ABI on the host (no GPU): the library loads, exports every entry point
include/moe_b200.h declares, and validates arguments before any launch."""
import ctypes

import numpy as np
import os
import re
import subprocess

import pytest

import prefill_moe_route_b200 as moe
from conftest import ROOT, read_golden
from prefill_moe_route_b200.synth import WORKLOADS

HEADER = os.path.join(ROOT, "include", "moe_b200.h")


def _declared():
    text = open(HEADER).read()
    return re.findall(r"MOE_API\s+[\w\s\*]*?\b(moe_\w+)\s*\(", text)


def test_library_exports_every_declared_entry_point():
    names = _declared()
    assert len(names) >= 8
    lib = moe.load()
    for n in names:
        assert hasattr(lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", moe.library_path()], capture_output=True, text=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    assert set(names) <= exported
    assert all(n.startswith("moe_") for n in exported)        # nothing else leaks


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workspace_size_and_layout(name):
    sh = WORKLOADS[name].shape()
    size = moe.moe_workspace_size(sh)
    lay = moe.moe_workspace_layout(sh)
    assert lay["total_bytes"] == size
    P = sh["M"] * sh["topk"]
    offs = [lay[k] for k in ("status", "topk_ids", "topk_w", "counts", "offsets", "sorted_pairs", "inv", "midq", "midqs")]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert lay["midqs"] - lay["midq"] >= P * sh["I"]
    assert size >= lay["midqs"] + P * (sh["I"] // 128) * 4


def test_mid_handoff_sizes_match_the_page():
    """The FP8 mid hand-off of "glm53: FP8 mid hand-off" at the page's shape
    (top-9, I = 512): mid as f32 is 74/147 KB at 4/8 rows; FP8 bytes plus one
    fp32 scale per 128-block are 19/38 KB; 8 rows hold 288 blocks."""
    for rows, f32_kb, fp8_kb, blocks in read_golden("mid_handoff_sizes.txt"):
        M = int(rows)
        sh = dict(M=M, H=6144, I=512, E=257, topk=9, routed_scale=1.0, wfmt=moe.MOE_W_MXFP4)
        lay = moe.moe_workspace_layout(sh)
        P = M * 9
        midq_bytes = lay["midqs"] - lay["midq"]               # 256-aligned region
        assert midq_bytes == -(-P * 512 // 256) * 256
        fp8_bytes = P * 512 + P * (512 // 128) * 4
        assert round(fp8_bytes / 1000) == int(fp8_kb)
        assert round(P * 512 * 4 / 1000) == int(f32_kb)
        assert fp8_bytes * 4 < P * 512 * 4 * 1.05 and P * 512 * 4 / (P * 512) == 4  # "a quarter of the bytes"
        if blocks != "-":
            assert P * 512 // 128 == int(blocks)


@pytest.mark.parametrize("bad,code", [
    (dict(M=0), moe.MOE_ERR_INVALID_ARG),
    (dict(I=200), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=384), moe.MOE_ERR_UNSUPPORTED),          # MXFP4 needs H % 256
    (dict(topk=17), moe.MOE_ERR_UNSUPPORTED),
    (dict(E=513), moe.MOE_ERR_UNSUPPORTED),
    (dict(topk=9, E=8), moe.MOE_ERR_UNSUPPORTED),
    (dict(wfmt=3), moe.MOE_ERR_INVALID_ARG),
])
def test_shape_validation(bad, code):
    sh = dict(WORKLOADS["tiny"].shape(), **bad)
    n = ctypes.c_size_t(0)
    rc = moe.load().moe_workspace_size(ctypes.byref(moe.MoeShape(**sh)), ctypes.byref(n))
    assert rc == code


def test_null_pointers_rejected_before_any_launch():
    sh = WORKLOADS["tiny"].shape()
    rc = moe.moe_forward(sh, None, None, None, None, None, None, None, None, None, 0, stream=0, check=False)
    assert rc == moe.MOE_ERR_INVALID_ARG
    rc = moe.moe_route(sh, None, None, None, None, stream=0, check=False)
    assert rc == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_quantize_mxfp4(None, 1, 32, None, None, stream=0, check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_quantize_fp8_block128(None, 1, 128, 128, None, None, stream=0, check=False) == moe.MOE_ERR_INVALID_ARG
    rc = moe.moe_forward_routed(sh, None, None, None, None, None, None, None, None, None, 0, stream=0, check=False)
    assert rc == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_pack_mxfp4_scales(None, 1, 128, 128, None, stream=0, check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_pack_mxfp4_scales(16, 1, 96, 128, 4096, stream=0, check=False) == moe.MOE_ERR_INVALID_ARG
    assert moe.moe_pack_mxfp4_scales(16, 1, 128, 128, 32, stream=0, check=False) == moe.MOE_ERR_INVALID_ARG  # overlap
    # misaligned pointers are rejected on the host too
    rc = moe.moe_forward(sh, 16, 16, None, 48, 16, 16, 16, 64, 16, 1 << 20, stream=0, check=False)
    assert rc == moe.MOE_ERR_INVALID_ARG


def test_packed_scale_order_is_the_tensor_core_word_order():
    """The packed layout puts row r of a 128-row tile in 32-bit word
    4 * (r % 32) + r // 32 of its 512-byte block (the order in which the
    tensor cores' 32 x 128-bit scale copy reads 128 rows of 4 scales), and
    the 4 scales of a word in column order; blocks run along K first."""
    from checks import pack_mx_scales
    rows, K = 256, 512
    s = np.arange(rows * K // 32, dtype=np.int64).reshape(rows, K // 32)   # scale id = r * K/32 + col
    src = (s % 251).astype(np.uint8)
    packed = pack_mx_scales(src).reshape(-1)
    for r in (0, 1, 31, 32, 33, 127, 128, 200, 255):
        for col in (0, 1, 3, 4, 7, 15):
            tile, rr = divmod(r, 128)
            grp, j = divmod(col, 4)
            byte = ((tile * (K // 128) + grp) * 512) + 16 * (rr % 32) + 4 * (rr // 32) + j
            assert packed[byte] == src[r, col]
    assert sorted(packed.tolist()) == sorted(src.reshape(-1).tolist())   # a permutation


def test_launches_per_call_needs_a_device():
    """A host-only query, but it answers for a device; without one (this CPU
    container) the index is out of range and the call says so."""
    sh = moe.MoeShape(**WORKLOADS["decode_tp8"].shape())
    n = ctypes.c_int32(-7)
    rc = moe.load().moe_launches_per_call(ctypes.byref(sh), 0, ctypes.byref(n))
    assert rc in (moe.MOE_OK, moe.MOE_ERR_INVALID_ARG)
    if rc == moe.MOE_OK:
        assert n.value in (1, 6)
    assert moe.load().moe_launches_per_call(None, 0, ctypes.byref(n)) == moe.MOE_ERR_INVALID_ARG


def test_tensor_probe_rejects_bad_arguments_before_any_launch():
    import ctypes
    L = moe.load()
    tf, mpc = ctypes.c_double(0.0), ctypes.c_double(0.0)
    for kind, iters in ((7, 100), (-1, 100), (moe.MOE_PROBE_FP8, 0), (moe.MOE_PROBE_FP8, 100001)):
        assert L.moe_probe_tensor_peak(kind, iters, ctypes.byref(tf), ctypes.byref(mpc), None) == moe.MOE_ERR_INVALID_ARG
    assert L.moe_probe_tensor_peak(moe.MOE_PROBE_FP8, 100, None, ctypes.byref(mpc), None) == moe.MOE_ERR_INVALID_ARG
