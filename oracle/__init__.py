"""CPU oracle of the quantized routed-expert MoE call (ctypes over moe_oracle.c).

TEST INFRASTRUCTURE ONLY: tests/, ``__graft_entry__.smoke()`` and the CPU legs
of ``bench.py`` may import this package; the product package
``prefill_moe_route_b200`` never does, and shares no code with it.

Every wrapper here only marshals numpy arrays; the arithmetic is in
``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libmoe_oracle.so")
_lib = None

W_MXFP4 = 1
W_FP8_BLOCK128 = 2


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into libmoe_oracle.so beside it."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(os.path.join(_HERE, "moe_oracle.h"))):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", _LIB_PATH + ".tmp", _SRC, "-lm"]
    subprocess.check_call(cmd, cwd=_HERE)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


class _Shape(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("wfmt", ctypes.c_int32)]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u8, i32, f32, f64, i64 = (ctypes.c_uint8, ctypes.c_int32, ctypes.c_float,
                                  ctypes.c_double, ctypes.c_int64)
        P = ctypes.c_void_p
        L.orc_e2m1_value.restype = f64; L.orc_e2m1_value.argtypes = [u8]
        L.orc_e2m1_encode.restype = u8; L.orc_e2m1_encode.argtypes = [f64]
        L.orc_e4m3_value.restype = f64; L.orc_e4m3_value.argtypes = [u8]
        L.orc_e4m3_encode.restype = u8; L.orc_e4m3_encode.argtypes = [f64]
        L.orc_e8m0_value.restype = f64; L.orc_e8m0_value.argtypes = [u8]
        L.orc_bf16_encode.restype = ctypes.c_uint16; L.orc_bf16_encode.argtypes = [f32]
        L.orc_bf16_value.restype = f32; L.orc_bf16_value.argtypes = [ctypes.c_uint16]
        L.orc_mx_scale_code.restype = u8; L.orc_mx_scale_code.argtypes = [f32]
        L.orc_pow2_scale_e4m3.restype = f32; L.orc_pow2_scale_e4m3.argtypes = [f32]
        L.orc_quant_mxfp4.restype = None; L.orc_quant_mxfp4.argtypes = [P, i64, i32, P, P]
        L.orc_quant_fp8_block128.restype = None; L.orc_quant_fp8_block128.argtypes = [P, i32, i32, P, P]
        L.orc_quant_fp8_pow2_row.restype = None; L.orc_quant_fp8_pow2_row.argtypes = [P, i32, P, P]
        L.orc_exp_spec.restype = f32; L.orc_exp_spec.argtypes = [f32]
        L.orc_sigmoid_spec.restype = f32; L.orc_sigmoid_spec.argtypes = [f32]
        L.orc_route.restype = None; L.orc_route.argtypes = [i32, i32, i32, P, P, f32, P, P]
        L.orc_align.restype = None; L.orc_align.argtypes = [i32, i32, i32, P, P, P, P, P]
        L.orc_quant_act_row.restype = None; L.orc_quant_act_row.argtypes = [i32, P, i32, P, P]
        L.orc_set_threads.restype = ctypes.c_int; L.orc_set_threads.argtypes = [ctypes.c_int]
        L.orc_forward_tokens.restype = ctypes.c_int
        L.orc_forward_tokens.argtypes = [ctypes.POINTER(_Shape), P, P, P, P, P, P, P, i32, P, P, P, P, P]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- codecs
def e2m1_value(code: int) -> float: return lib().orc_e2m1_value(code)
def e2m1_encode(v: float) -> int: return lib().orc_e2m1_encode(v)
def e4m3_value(code: int) -> float: return lib().orc_e4m3_value(code)
def e4m3_encode(v: float) -> int: return lib().orc_e4m3_encode(v)
def e8m0_value(code: int) -> float: return lib().orc_e8m0_value(code)
def bf16_encode(v: float) -> int: return lib().orc_bf16_encode(v)
def bf16_value(b: int) -> float: return lib().orc_bf16_value(b)
def mx_scale_code(amax: float) -> int: return lib().orc_mx_scale_code(amax)
def pow2_scale_e4m3(amax: float) -> float: return lib().orc_pow2_scale_e4m3(amax)
def exp_spec(x: float) -> float: return lib().orc_exp_spec(x)
def sigmoid_spec(x: float) -> float: return lib().orc_sigmoid_spec(x)


def set_threads(n: int) -> int:
    """OpenMP threads of the oracle's loops (timing only); returns the previous count."""
    return lib().orc_set_threads(int(n))


def quant_mxfp4(w: np.ndarray):
    """[..., K] fp32 -> (packed u8 [..., K/2], scales u8 [..., K/32])."""
    w = _c(w, np.float32)
    K = w.shape[-1]
    rows = w.size // K
    q = np.empty(w.shape[:-1] + (K // 2,), np.uint8)
    s = np.empty(w.shape[:-1] + (K // 32,), np.uint8)
    lib().orc_quant_mxfp4(_p(w), rows, K, _p(q), _p(s))
    return q, s


def quant_fp8_block128(w: np.ndarray):
    """[..., R, K] fp32 -> (codes u8 [..., R, K], scales f32 [..., R/128, K/128])."""
    w = _c(w, np.float32)
    R, K = w.shape[-2:]
    lead = w.shape[:-2]
    q = np.empty(w.shape, np.uint8)
    s = np.empty(lead + (R // 128, K // 128), np.float32)
    wf = w.reshape(-1, R, K)
    qf = q.reshape(-1, R, K)
    sf = s.reshape(-1, R // 128, K // 128)
    for b in range(wf.shape[0]):
        lib().orc_quant_fp8_block128(_p(wf[b]), R, K, _p(qf[b]), _p(sf[b]))
    return q, s


def quant_fp8_pow2_row(v: np.ndarray):
    v = _c(v, np.float32)
    K = v.shape[-1]
    q = np.empty(K, np.uint8)
    s = np.empty(K // 128, np.float32)
    lib().orc_quant_fp8_pow2_row(_p(v), K, _p(q), _p(s))
    return q, s


def quant_act(wfmt: int, x_bf16: np.ndarray):
    """x bf16 bits [M, H] -> (q, s) as the format asks."""
    x = _c(x_bf16, np.uint16)
    M, H = x.shape
    if wfmt == W_MXFP4:
        q = np.empty((M, H // 2), np.uint8); s = np.empty((M, H // 32), np.uint8)
    else:
        q = np.empty((M, H), np.uint8); s = np.empty((M, H // 128), np.float32)
    for t in range(M):
        lib().orc_quant_act_row(wfmt, _p(x[t]), H, _p(q[t]), _p(s[t]))
    return q, s


def route(logits: np.ndarray, bias, k: int, routed_scale: float):
    logits = _c(logits, np.float32)
    M, E = logits.shape
    b = None if bias is None else _c(bias, np.float32)
    ids = np.empty((M, k), np.int32)
    w = np.empty((M, k), np.float32)
    lib().orc_route(M, E, k, _p(logits), _p(b), routed_scale, _p(ids), _p(w))
    return ids, w


def align(topk_ids: np.ndarray, E: int):
    ids = _c(topk_ids, np.int32)
    M, k = ids.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    sp = np.empty(M * k, np.int32)
    inv = np.empty(M * k, np.int32)
    lib().orc_align(M, k, E, _p(ids), _p(counts), _p(offsets), _p(sp), _p(inv))
    return counts, offsets, sp, inv


def forward_tokens(shape: dict, x, topk_ids, topk_w, w13, s13, w2, s2, tokens=None,
                   want_midq: bool = True):
    """Run the oracle forward on `tokens` (all tokens if None).

    Returns dict(midq [n*k, I] u8, midqs [n*k, I/128] f32, ref [n, H] f64,
    out [n, H] bf16 bits), pair rows in (token, slot) order.
    """
    sh = _Shape(shape["M"], shape["H"], shape["I"], shape["E"], shape["topk"],
                shape["routed_scale"], shape["wfmt"])
    M, H, I, k = shape["M"], shape["H"], shape["I"], shape["topk"]
    toks = None if tokens is None else _c(tokens, np.int32)
    n = M if toks is None else toks.size
    midq = np.empty((n * k, I), np.uint8) if want_midq else None
    midqs = np.empty((n * k, I // 128), np.float32) if want_midq else None
    ref = np.empty((n, H), np.float64)
    out = np.empty((n, H), np.uint16)
    arrs = [_c(x, np.uint16), _c(topk_ids, np.int32), _c(topk_w, np.float32),
            _c(w13, np.uint8), np.ascontiguousarray(s13), _c(w2, np.uint8), np.ascontiguousarray(s2)]
    rc = lib().orc_forward_tokens(ctypes.byref(sh), *[_p(a) for a in arrs], n, _p(toks),
                                  _p(midq), _p(midqs), _p(ref), _p(out))
    if rc != 0:
        raise ValueError("orc_forward_tokens rejected its arguments")
    return {"midq": midq, "midqs": midqs, "ref": ref, "out": out}
