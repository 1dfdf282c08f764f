"""Device-side setup of one MoE problem: torch allocations + calls into the C ABI.

Used by the tests, ``bench.py`` and ``__graft_entry__.smoke()``.  Weights are
drawn per expert as fp32 (``synth.Inputs``), moved to the GPU and quantized
there by the library's own ``moe_quantize_*`` kernels; an optional callback
sees each expert's fp32 draw so a checker can quantize it independently.
MXFP4 scales are kept both row-major (``s13``/``s2``, the quantizer's output,
what a checker compares) and packed for ``moe_forward`` (``sf13``/``sf2``).
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

from . import (MOE_W_MXFP4, moe_forward, moe_get_status, moe_pack_mxfp4_scales, moe_quantize_fp8_block128,
               moe_quantize_mxfp4, moe_workspace_init, moe_workspace_layout, moe_workspace_size)
from .synth import Inputs, Workload


def _expert_draws(inputs: Inputs, E: int):
    """(w13, w2) fp32 draws of experts 0..E-1 in order.  Each expert has its own
    random stream, so the draws run on a few host threads (numpy releases the
    GIL while it fills), at most a small window ahead of the consumer."""
    workers = max(1, min(16, (os.cpu_count() or 1)))
    with ThreadPoolExecutor(max_workers=workers) as pool:
        draw = lambda e: (inputs.w13(e), inputs.w2(e))
        pending = [pool.submit(draw, e) for e in range(min(E, 2 * workers))]
        for e in range(E):
            f13, f2 = pending[e].result()
            pending[e] = None
            if e + 2 * workers < E:
                pending.append(pool.submit(draw, e + 2 * workers))
            yield f13, f2


class DeviceMoE:
    """Inputs, quantized weights, output and workspace of one problem on one GPU."""

    def __init__(self, wl: Workload, inputs: Inputs, device="cuda:0", on_expert=None):
        self.wl = wl
        self.device = torch.device(device)
        self.shape = wl.shape()
        M, H, I, E = wl.M, wl.H, wl.I, wl.E
        dev = self.device
        u8, f32 = torch.uint8, torch.float32
        mx = wl.wfmt == MOE_W_MXFP4
        if mx:
            self.w13 = torch.empty((E, 2 * I, H // 2), dtype=u8, device=dev)
            self.s13 = torch.empty((E, 2 * I, H // 32), dtype=u8, device=dev)
            self.w2 = torch.empty((E, H, I // 2), dtype=u8, device=dev)
            self.s2 = torch.empty((E, H, I // 32), dtype=u8, device=dev)
        else:
            self.w13 = torch.empty((E, 2 * I, H), dtype=u8, device=dev)
            self.s13 = torch.empty((E, 2 * I // 128, H // 128), dtype=f32, device=dev)
            self.w2 = torch.empty((E, H, I), dtype=u8, device=dev)
            self.s2 = torch.empty((E, H // 128, I // 128), dtype=f32, device=dev)
        stream = torch.cuda.current_stream(dev)
        with torch.cuda.device(dev):
            for e, (f13, f2) in enumerate(_expert_draws(inputs, E)):
                if on_expert is not None:
                    on_expert(e, f13, f2)
                g13 = torch.from_numpy(f13).to(dev, non_blocking=False)
                g2 = torch.from_numpy(f2).to(dev, non_blocking=False)
                if mx:
                    moe_quantize_mxfp4(g13, 2 * I, H, self.w13[e], self.s13[e], stream)
                    moe_quantize_mxfp4(g2, H, I, self.w2[e], self.s2[e], stream)
                else:
                    moe_quantize_fp8_block128(g13, 1, 2 * I, H, self.w13[e], self.s13[e], stream)
                    moe_quantize_fp8_block128(g2, 1, H, I, self.w2[e], self.s2[e], stream)
                del g13, g2
            if mx:
                self.sf13 = torch.empty_like(self.s13)
                self.sf2 = torch.empty_like(self.s2)
                moe_pack_mxfp4_scales(self.s13, E, 2 * I, H, self.sf13, stream)
                moe_pack_mxfp4_scales(self.s2, E, H, I, self.sf2, stream)
            else:
                self.sf13, self.sf2 = self.s13, self.s2
            torch.cuda.synchronize(dev)
        self.set_activations(inputs.x, inputs.logits, inputs.bias)
        self.out = torch.empty((M, H), dtype=torch.int16, device=dev)
        self.ws_bytes = moe_workspace_size(self.shape)
        self.workspace = torch.empty(self.ws_bytes, dtype=u8, device=dev)
        moe_workspace_init(self.workspace, self.ws_bytes, stream)
        self.layout = moe_workspace_layout(self.shape)

    def set_activations(self, x_bf16: np.ndarray, logits: np.ndarray, bias):
        dev = self.device
        self.x = torch.from_numpy(np.ascontiguousarray(x_bf16).view(np.int16)).to(dev)
        self.logits = torch.from_numpy(np.ascontiguousarray(logits, np.float32)).to(dev)
        self.bias = None if bias is None else torch.from_numpy(np.ascontiguousarray(bias, np.float32)).to(dev)

    def forward(self, stream=None, out=None, x=None, logits=None):
        return moe_forward(self.shape, self.x if x is None else x, self.logits if logits is None else logits,
                           self.bias, self.w13, self.sf13, self.w2, self.sf2,
                           self.out if out is None else out, self.workspace, self.ws_bytes, stream)

    def status(self, stream=None):
        return moe_get_status(self.workspace, stream)

    def status_words(self):
        """Raw status region: [0] status, [1] route arrival counter, [2] first timed-out wait."""
        off = self.layout["status"]
        return self.workspace[off:off + 16].cpu().numpy().view(np.int32).copy()

    # ---- debug taps (copies to host numpy)
    def _tap(self, name: str, dtype, count: int) -> np.ndarray:
        off = self.layout[name]
        nbytes = count * np.dtype(dtype).itemsize
        return self.workspace[off:off + nbytes].cpu().numpy().view(dtype).copy()

    def taps(self) -> dict:
        wl = self.wl
        P = wl.M * wl.topk
        return {
            "topk_ids": self._tap("topk_ids", np.int32, P).reshape(wl.M, wl.topk),
            "topk_w": self._tap("topk_w", np.float32, P).reshape(wl.M, wl.topk),
            "counts": self._tap("counts", np.int32, wl.E),
            "offsets": self._tap("offsets", np.int32, wl.E + 1),
            "sorted_pairs": self._tap("sorted_pairs", np.int32, P),
            "inv": self._tap("inv", np.int32, P),
            "midq": self._tap("midq", np.uint8, P * wl.I).reshape(P, wl.I),
            "midqs": self._tap("midqs", np.float32, P * (wl.I // 128)).reshape(P, wl.I // 128),
        }

    def out_bits(self) -> np.ndarray:
        return self.out.cpu().numpy().view(np.uint16)

    def weights_host(self):
        return tuple(t.cpu().numpy() for t in (self.w13, self.s13, self.w2, self.s2))
