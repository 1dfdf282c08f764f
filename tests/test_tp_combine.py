"""The tensor-parallel split on the CPU: two gloo ranks each take a
128-aligned slice of every expert's intermediate dimension
(prefill_moe_route_b200.tp.slice_expert_weights), compute the oracle's result
on their slice with the shared routing, and all-reduce the partial outputs;
the sum equals the oracle's unsplit call (the mid blocks of 128 and the
weight blocks are never cut, so only the summation order differs)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from prefill_moe_route_b200.synth import W_FP8_BLOCK128, W_MXFP4, to_bf16_bits
from prefill_moe_route_b200.tp import slice_expert_weights


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(wfmt):
    rng = np.random.default_rng(61 + wfmt)
    M, H, I, E, k = 5, 256, 256, 6, 2
    x = to_bf16_bits(rng.standard_normal((M, H)).astype(np.float32))
    logits = rng.standard_normal((M, E)).astype(np.float32)
    f13 = (rng.standard_normal((E, 2 * I, H)) * 0.02).astype(np.float32)
    f2 = (rng.standard_normal((E, H, I)) * 0.02).astype(np.float32)
    if wfmt == W_MXFP4:
        w = (*oracle.quant_mxfp4(f13), *oracle.quant_mxfp4(f2))
    else:
        w = (*oracle.quant_fp8_block128(f13), *oracle.quant_fp8_block128(f2))
    return dict(M=M, H=H, I=I, E=E, topk=k, routed_scale=2.5, wfmt=wfmt), x, logits, w


def _rank(rank, world, port, wfmt, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        shape, x, logits, w = _problem(wfmt)
        ids, tw = oracle.route(logits, None, shape["topk"], shape["routed_scale"])
        parts = slice_expert_weights(*[torch.from_numpy(a) for a in w], wfmt, shape["I"], rank, world)
        sub = dict(shape, I=shape["I"] // world)
        res = oracle.forward_tokens(sub, x, ids, tw, *[p.numpy() for p in parts])
        partial = torch.from_numpy(res["ref"].copy())
        dist.all_reduce(partial, op=dist.ReduceOp.SUM)
        out[rank] = partial.numpy()
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("wfmt", [W_MXFP4, W_FP8_BLOCK128], ids=["mxfp4", "fp8"])
def test_two_rank_split_sums_to_the_unsplit_call(wfmt):
    world, port = 2, _free_port()
    out = mp.Manager().dict()
    mp.spawn(_rank, args=(world, port, wfmt, out), nprocs=world, join=True)
    shape, x, logits, w = _problem(wfmt)
    ids, tw = oracle.route(logits, None, shape["topk"], shape["routed_scale"])
    ref = oracle.forward_tokens(shape, x, ids, tw, *w)["ref"]
    for r in range(world):
        assert np.allclose(out[r], ref, rtol=1e-12, atol=1e-14)
    assert np.array_equal(out[0], out[1])


def test_slices_reassemble_the_weights():
    rng = np.random.default_rng(3)
    E, H, I = 2, 256, 512
    for wfmt in (W_MXFP4, W_FP8_BLOCK128):
        if wfmt == W_MXFP4:
            full = [torch.from_numpy(rng.integers(0, 255, s, dtype=np.uint8)) for s in
                    ((E, 2 * I, H // 2), (E, 2 * I, H // 32), (E, H, I // 2), (E, H, I // 32))]
        else:
            full = [torch.from_numpy(rng.integers(0, 255, (E, 2 * I, H), dtype=np.uint8)),
                    torch.from_numpy(rng.random((E, 2 * I // 128, H // 128)).astype(np.float32)),
                    torch.from_numpy(rng.integers(0, 255, (E, H, I), dtype=np.uint8)),
                    torch.from_numpy(rng.random((E, H // 128, I // 128)).astype(np.float32))]
        sl = [slice_expert_weights(*full, wfmt, I, r, 4) for r in range(4)]
        n = I // 4
        for r in range(4):
            g = 1 if wfmt == W_MXFP4 else 128      # rows per scale row of w13
            assert torch.equal(sl[r][0][:, :n], full[0][:, r * n:(r + 1) * n])
            assert torch.equal(sl[r][0][:, n:], full[0][:, I + r * n:I + (r + 1) * n])
            assert torch.equal(sl[r][1][:, :n // g], full[1][:, r * n // g:(r + 1) * n // g])
        w2 = torch.cat([s[2] for s in sl], 2)
        s2 = torch.cat([s[3] for s in sl], 2)
        assert torch.equal(w2, full[2]) and torch.equal(s2, full[3])
    with pytest.raises(ValueError):
        slice_expert_weights(*full, W_FP8_BLOCK128, 256, 0, 4)      # 64-wide slices would cut blocks
