"""Test helper: one moe_forward_static call on a DeviceMoE problem's inputs."""
import numpy as np
import torch

import prefill_moe_route_b200 as moe


def static_call(dev, fill=0):
    """Runs moe_forward_static on dev's inputs and weights; returns out as bf16 bits."""
    out = torch.empty_like(dev.out)
    out.fill_(fill)
    rc = moe.moe_forward_static(dev.shape, dev.x, dev.logits, dev.bias, dev.w13, dev.sf13, dev.w2, dev.sf2, out,
                                check=False)
    assert rc == moe.MOE_OK, moe.moe_last_error()
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint16).copy()
