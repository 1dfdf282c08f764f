"""Tensor-parallel MoE call over T ranks: each rank holds a 128-aligned slice
of every expert's intermediate dimension I (the pages' TP4/TP8 rank slices,
"[HIP] IQ2R: GLM-5.3 packed MoE path for TP4/TP8 on gfx950", Technical
Details).  Every rank routes the same logits, runs moe_forward_partial on its
slice (fp32 partial sums of the output), the partials are summed across the
ranks by one all-reduce (NCCL over NVLink on GPUs; the pages' ranks exchange
partial sums, "glm53: FP8 mid hand-off", Accuracy Tests), and moe_round_bf16
rounds the sum to the bf16 output.

Argument marshalling and the collective only: the MoE arithmetic runs in the
library's kernels.
"""
from __future__ import annotations

from . import MOE_W_MXFP4, moe_forward_partial, moe_round_bf16


def slice_expert_weights(w13, s13, w2, s2, wfmt: int, I: int, rank: int, world: int):
    """The rank's share of the quantized experts (torch tensors, host or device).

    w13 [E][2I][...] rows [0, I) gate, [I, 2I) up -> the slice's gate rows then
    its up rows; w2 [E][H][I ...] -> the slice's columns.  Scales follow their
    payload: MXFP4 row-major E8M0 [E][rows][K/32] (pack them afterwards for
    moe_forward_partial), block FP8 [E][rows/128][K/128].  I / world must be a
    multiple of 128, so quantization blocks are never cut."""
    import torch
    if I % world or (I // world) % 128:
        raise ValueError("each rank's slice of I must be a multiple of 128")
    n = I // world
    a, b = rank * n, (rank + 1) * n
    if wfmt == MOE_W_MXFP4:
        w13r = torch.cat([w13[:, a:b], w13[:, I + a:I + b]], 1).contiguous()
        s13r = torch.cat([s13[:, a:b], s13[:, I + a:I + b]], 1).contiguous()
        w2r = w2[:, :, a // 2:b // 2].contiguous()
        s2r = s2[:, :, a // 32:b // 32].contiguous()
    else:
        w13r = torch.cat([w13[:, a:b], w13[:, I + a:I + b]], 1).contiguous()
        s13r = torch.cat([s13[:, a // 128:b // 128], s13[:, (I + a) // 128:(I + b) // 128]], 1).contiguous()
        w2r = w2[:, :, a:b].contiguous()
        s2r = s2[:, :, a // 128:b // 128].contiguous()
    return w13r, s13r, w2r, s2r


def tp_forward(shape, x, logits, bias, w13, w13_scales, w2, w2_scales, out, partial, workspace, ws_bytes: int,
               group=None, stream=None):
    """One rank's step of the tensor-parallel call: its partial, the all-reduce
    (sum) over `group`, the bf16 rounding into `out`.  `shape` is the rank's
    (its I is the slice width); `partial` an fp32 [M][H] buffer."""
    import torch.distributed as dist
    moe_forward_partial(shape, x, logits, bias, w13, w13_scales, w2, w2_scales, partial, workspace, ws_bytes, stream)
    if group is not None or (dist.is_available() and dist.is_initialized()):
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    moe_round_bf16(partial, out, partial.numel(), stream)
