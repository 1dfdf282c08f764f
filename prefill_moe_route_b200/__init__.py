"""Python binding of libmoe_b200.so (the C ABI in include/moe_b200.h).

Argument marshalling only: every step of the MoE call runs in the library's
CUDA kernels.  Tensors may be passed as torch tensors (their ``data_ptr()`` is
used) or as integer device addresses; streams as ``torch.cuda.Stream``, a raw
``cudaStream_t`` integer, or None for torch's current stream.

The library is loaded on first use; calling an entry point without the built
library raises ``RuntimeError`` (there is no fallback implementation).
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "MOE_OK", "MOE_ERR_INVALID_ARG", "MOE_ERR_UNSUPPORTED", "MOE_ERR_WORKSPACE",
    "MOE_ERR_DEVICE_MISMATCH", "MOE_ERR_CUDA", "MOE_ERR_DEVICE_TIMEOUT",
    "MOE_W_MXFP4", "MOE_W_FP8_BLOCK128", "MoeError", "MoeShape", "library_path", "load",
    "moe_last_error", "moe_workspace_size", "moe_workspace_layout", "moe_workspace_init", "moe_route",
    "moe_forward", "moe_forward_routed", "moe_forward_partial", "moe_round_bf16", "moe_forward_timed", "moe_forward_static", "moe_get_status_static", "moe_launches_per_call", "MOE_STATIC_SCRATCH_BYTES", "moe_get_status", "moe_quantize_mxfp4", "moe_pack_mxfp4_scales", "moe_quantize_fp8_block128",
    "moe_probe_tensor_peak", "MOE_PROBE_FP8", "MOE_PROBE_FP4", "MOE_PROBE_BF16",
]

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_DEVICE_MISMATCH = -4
MOE_ERR_CUDA = -5
MOE_ERR_DEVICE_TIMEOUT = -6
MOE_W_MXFP4 = 1
MOE_W_FP8_BLOCK128 = 2
MOE_PROBE_FP8 = 0
MOE_PROBE_FP4 = 1
MOE_PROBE_BF16 = 2

_NAMES = {0: "MOE_OK", -1: "MOE_ERR_INVALID_ARG", -2: "MOE_ERR_UNSUPPORTED", -3: "MOE_ERR_WORKSPACE",
          -4: "MOE_ERR_DEVICE_MISMATCH", -5: "MOE_ERR_CUDA", -6: "MOE_ERR_DEVICE_TIMEOUT"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmoe_b200.so")
_lib = None


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        detail = moe_last_error()
        super().__init__(f"{where} returned {_NAMES.get(code, code)}" + (f" ({detail})" if detail else ""))
        self.code = code


class MoeShape(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("H", ctypes.c_int32), ("I", ctypes.c_int32),
                ("E", ctypes.c_int32), ("topk", ctypes.c_int32),
                ("routed_scale", ctypes.c_float), ("wfmt", ctypes.c_int32)]

    @classmethod
    def of(cls, M, H, I, E, topk, routed_scale, wfmt):
        return cls(M, H, I, E, topk, routed_scale, wfmt)


class _Layout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_uint64) for n in
                ("status", "topk_ids", "topk_w", "counts", "offsets", "sorted_pairs", "inv",
                 "midq", "midqs", "total_bytes")]


def library_path() -> str:
    return _LIB_PATH


def load():
    """Load libmoe_b200.so (once)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is not built; run `python -m prefill_moe_route_b200.build`")
    L = ctypes.CDLL(_LIB_PATH)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    SH = ctypes.POINTER(MoeShape)
    sig = {
        "moe_workspace_size": [SH, ctypes.POINTER(SZ)],
        "moe_workspace_layout": [SH, ctypes.POINTER(_Layout)],
        "moe_workspace_init": [P, SZ, P],
        "moe_route": [SH, P, P, P, P, P],
        "moe_forward": [SH, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_forward_routed": [SH, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_forward_partial": [SH, P, P, P, P, P, P, P, P, P, SZ, P],
        "moe_round_bf16": [P, P, I64, P],
        "moe_forward_timed": [SH, P, P, P, P, P, P, P, P, P, SZ, P, ctypes.POINTER(P)],
        "moe_forward_static": [SH, P, P, P, P, P, P, P, P, P],
        "moe_get_status": [P, P, ctypes.POINTER(I32)],
        "moe_get_status_static": [P, ctypes.POINTER(I32)],
        "moe_launches_per_call": [SH, I32, ctypes.POINTER(I32)],
        "moe_quantize_mxfp4": [P, I64, I32, P, P, P],
        "moe_pack_mxfp4_scales": [P, I64, I32, I32, P, P],
        "moe_quantize_fp8_block128": [P, I64, I32, I32, P, P, P],
        "moe_probe_tensor_peak": [I32, I32, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double), P],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    L.moe_last_error.argtypes = []
    L.moe_last_error.restype = ctypes.c_char_p
    _lib = L
    return L


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _ret(rc: int, where: str, check: bool) -> int:
    if check and rc != MOE_OK:
        raise MoeError(rc, where)
    return rc


def _shape(shape):
    if isinstance(shape, MoeShape):
        return shape
    return MoeShape(shape["M"], shape["H"], shape["I"], shape["E"], shape["topk"],
                    shape["routed_scale"], shape["wfmt"])


def moe_last_error() -> str:
    """Text of the last failed library call on this thread."""
    return load().moe_last_error().decode(errors="replace")


def moe_workspace_size(shape) -> int:
    n = ctypes.c_size_t(0)
    _ret(load().moe_workspace_size(ctypes.byref(_shape(shape)), ctypes.byref(n)), "moe_workspace_size", True)
    return n.value


def moe_workspace_layout(shape) -> dict:
    lay = _Layout()
    _ret(load().moe_workspace_layout(ctypes.byref(_shape(shape)), ctypes.byref(lay)), "moe_workspace_layout", True)
    return {n: getattr(lay, n) for n, _ in _Layout._fields_}


def moe_workspace_init(workspace, ws_bytes: int, stream=None, check: bool = True) -> int:
    return _ret(load().moe_workspace_init(_ptr(workspace), ws_bytes, _stream(stream)), "moe_workspace_init", check)


def moe_route(shape, logits, bias, topk_ids, topk_w, stream=None, check: bool = True) -> int:
    rc = load().moe_route(ctypes.byref(_shape(shape)), _ptr(logits), _ptr(bias), _ptr(topk_ids),
                          _ptr(topk_w), _stream(stream))
    return _ret(rc, "moe_route", check)


def moe_forward(shape, x, logits, bias, w13, w13_scales, w2, w2_scales, out, workspace, ws_bytes: int,
                stream=None, check: bool = True) -> int:
    rc = load().moe_forward(ctypes.byref(_shape(shape)), _ptr(x), _ptr(logits), _ptr(bias), _ptr(w13),
                            _ptr(w13_scales), _ptr(w2), _ptr(w2_scales), _ptr(out), _ptr(workspace),
                            ws_bytes, _stream(stream))
    return _ret(rc, "moe_forward", check)


def moe_forward_routed(shape, x, topk_ids, topk_w, w13, w13_scales, w2, w2_scales, out, workspace, ws_bytes: int,
                       stream=None, check: bool = True) -> int:
    """moe_forward with the caller's expert selection (int32 ids, fp32 weights, [M][topk]) instead of logits."""
    rc = load().moe_forward_routed(ctypes.byref(_shape(shape)), _ptr(x), _ptr(topk_ids), _ptr(topk_w), _ptr(w13),
                                   _ptr(w13_scales), _ptr(w2), _ptr(w2_scales), _ptr(out), _ptr(workspace),
                                   ws_bytes, _stream(stream))
    return _ret(rc, "moe_forward_routed", check)


def moe_forward_partial(shape, x, logits, bias, w13, w13_scales, w2, w2_scales, out_partial, workspace,
                        ws_bytes: int, stream=None, check: bool = True) -> int:
    """One tensor-parallel rank's share: its I-slice of every expert, fp32 [M][H] partial sums out."""
    rc = load().moe_forward_partial(ctypes.byref(_shape(shape)), _ptr(x), _ptr(logits), _ptr(bias), _ptr(w13),
                                    _ptr(w13_scales), _ptr(w2), _ptr(w2_scales), _ptr(out_partial),
                                    _ptr(workspace), ws_bytes, _stream(stream))
    return _ret(rc, "moe_forward_partial", check)


def moe_round_bf16(src, out, n: int, stream=None, check: bool = True) -> int:
    """bf16 (round to nearest even) of n fp32 values (n % 8 == 0)."""
    return _ret(load().moe_round_bf16(_ptr(src), _ptr(out), n, _stream(stream)), "moe_round_bf16", check)


def moe_forward_timed(shape, x, logits, bias, w13, w13_scales, w2, w2_scales, out, workspace, ws_bytes: int,
                      events, stream=None, check: bool = True) -> int:
    """moe_forward recording 5 CUDA events (torch.cuda.Event or raw handles) around its kernels."""
    handles = (ctypes.c_void_p * 5)(*[e if isinstance(e, int) else e.cuda_event for e in events])
    rc = load().moe_forward_timed(ctypes.byref(_shape(shape)), _ptr(x), _ptr(logits), _ptr(bias), _ptr(w13),
                                  _ptr(w13_scales), _ptr(w2), _ptr(w2_scales), _ptr(out), _ptr(workspace),
                                  ws_bytes, _stream(stream), handles)
    return _ret(rc, "moe_forward_timed", check)


MOE_STATIC_SCRATCH_BYTES = 8 << 20


def moe_forward_static(shape, x, logits, bias, w13, w13_scales, w2, w2_scales, out, stream=None,
                       check: bool = True) -> int:
    """moe_forward without a caller workspace: the library's fixed static scratch is used
    (see include/moe_b200.h for its limits and for who needs it)."""
    rc = load().moe_forward_static(ctypes.byref(_shape(shape)), _ptr(x), _ptr(logits), _ptr(bias), _ptr(w13),
                                   _ptr(w13_scales), _ptr(w2), _ptr(w2_scales), _ptr(out), _stream(stream))
    return _ret(rc, "moe_forward_static", check)


def moe_get_status_static(stream=None):
    """Status word of the static scratch of moe_forward_static: (return code, device status word)."""
    v = ctypes.c_int32(0)
    rc = load().moe_get_status_static(_stream(stream), ctypes.byref(v))
    return rc, v.value


def moe_probe_tensor_peak(kind: int, iters: int = 4000, stream=None):
    """Measured tensor-core throughput for one MMA kind: (TFLOP/s over the
    GPU, MACs per SM clock).  Synchronizes the stream."""
    tf, mpc = ctypes.c_double(0.0), ctypes.c_double(0.0)
    _ret(load().moe_probe_tensor_peak(kind, iters, ctypes.byref(tf), ctypes.byref(mpc), _stream(stream)),
         "moe_probe_tensor_peak", True)
    return tf.value, mpc.value


def moe_launches_per_call(shape, device: int = 0) -> int:
    """Kernels one moe_forward of this shape launches on `device` (1: the single decode-sized kernel)."""
    v = ctypes.c_int32(0)
    _ret(load().moe_launches_per_call(ctypes.byref(_shape(shape)), device, ctypes.byref(v)),
         "moe_launches_per_call", True)
    return v.value


def moe_get_status(workspace, stream=None):
    """Returns (return code, device status word)."""
    v = ctypes.c_int32(0)
    rc = load().moe_get_status(_ptr(workspace), _stream(stream), ctypes.byref(v))
    return rc, v.value


def moe_quantize_mxfp4(w, rows: int, K: int, q, scales, stream=None, check: bool = True) -> int:
    rc = load().moe_quantize_mxfp4(_ptr(w), rows, K, _ptr(q), _ptr(scales), _stream(stream))
    return _ret(rc, "moe_quantize_mxfp4", check)


def moe_pack_mxfp4_scales(scales, batch: int, rows: int, K: int, packed, stream=None, check: bool = True) -> int:
    """Row-major MXFP4 E8M0 scales -> the packed layout moe_forward reads (include/moe_b200.h)."""
    rc = load().moe_pack_mxfp4_scales(_ptr(scales), batch, rows, K, _ptr(packed), _stream(stream))
    return _ret(rc, "moe_pack_mxfp4_scales", check)


def moe_quantize_fp8_block128(w, batch: int, rows: int, K: int, q, scales, stream=None,
                              check: bool = True) -> int:
    rc = load().moe_quantize_fp8_block128(_ptr(w), batch, rows, K, _ptr(q), _ptr(scales), _stream(stream))
    return _ret(rc, "moe_quantize_fp8_block128", check)
