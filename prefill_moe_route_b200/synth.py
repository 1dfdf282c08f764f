"""Seeded synthetic inputs for the routed-expert MoE call.

This module is shared by the tests, the oracle harness and ``bench.py``.  It
draws numbers and holds none of the method's arithmetic: no routing, no
quantization, no contraction.  Quantized weights are produced from the fp32
draws by each side on its own (the library's ``moe_quantize_*`` kernels, the
oracle's C codecs).

Workloads (shapes and distributions of the five per-rank slices the MoE call
is measured on; the pages' shared-expert top-9 layer is not among them):

==================  ====  ====  ===  ==  ===  ======  =====  ==========================
name                M     H     E    k   I    format  scale  router logits
==================  ====  ====  ===  ==  ===  ======  =====  ==========================
tiny                4     512   8    2   256  mxfp4   1.0    N(0,1), bias N(0,0.1)
decode_tp8          4     6144  256  8   256  mxfp4   2.5    N(0,1) i.i.d.
decode_tp4_skew     16    6144  256  8   512  mxfp4   2.5    N(0,1) + 2.0 on 16 experts
prefill_tp8         1024  6144  256  8   256  mxfp4   2.5    N(0,1) i.i.d.
prefill_tp4_fp8     4096  6144  256  8   512  fp8     2.5    Zipf(1.1) Gumbel-top-k
==================  ====  ====  ===  ==  ===  ======  =====  ==========================

x ~ N(0,1) rounded to bf16; w13 [E, 2I, H] and w2 [E, H, I] ~ N(0, 0.02) fp32.
MEDIUM and CROSSOVER hold the medium-M workloads (M = 32..512, spread / hot /
mixed routing) and the decode sizes timed on both paths.
Every tensor has its own stream: ``SeedSequence([seed, tag, *index])`` with
PCG64, so one expert's weights can be drawn without drawing the others.
"""
from __future__ import annotations

import dataclasses

import numpy as np

W_MXFP4 = 1
W_FP8_BLOCK128 = 2

_TAGS = {"x": 1, "logits": 2, "bias": 3, "hot": 4, "perm": 5, "gumbel": 6, "w13": 7, "w2": 8, "hotset": 9}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    M: int
    H: int
    E: int
    topk: int
    I: int
    wfmt: int
    routed_scale: float
    logits: str           # "normal" | "skew16" | "zipf1.1" | "hot" | "mixed"
    bias: bool            # draw a N(0, 0.1) router bias

    def shape(self) -> dict:
        return dict(M=self.M, H=self.H, I=self.I, E=self.E, topk=self.topk,
                    routed_scale=self.routed_scale, wfmt=self.wfmt)

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    "tiny": Workload("tiny", 4, 512, 8, 2, 256, W_MXFP4, 1.0, "normal", True),
    "decode_tp8": Workload("decode_tp8", 4, 6144, 256, 8, 256, W_MXFP4, 2.5, "normal", False),
    "decode_tp4_skew": Workload("decode_tp4_skew", 16, 6144, 256, 8, 512, W_MXFP4, 2.5, "skew16", False),
    "prefill_tp8": Workload("prefill_tp8", 1024, 6144, 256, 8, 256, W_MXFP4, 2.5, "normal", False),
    "prefill_tp4_fp8": Workload("prefill_tp4_fp8", 4096, 6144, 256, 8, 512, W_FP8_BLOCK128, 2.5, "zipf1.1", False),
}


# The medium-M regime (the pages' M32..M256 rows, TP8 rank slice, MXFP4) under
# three routing patterns: spread (i.i.d. N(0,1) logits, as many distinct
# experts as the tokens pick), hot (all tokens on the same few experts) and
# mixed (half of the tokens hot).
MEDIUM = {f"medium_M{M}_{r}": Workload(f"medium_M{M}_{r}", M, 6144, 256, 8, 256, W_MXFP4, 2.5,
                                      "normal" if r == "spread" else r, False)
          for M in (32, 64, 128, 256, 512) for r in ("spread", "hot", "mixed")}

# Decode sizes on both paths: where the single-launch kernel and the grouped
# kernels cross over (M <= 16 runs either way).
CROSSOVER = {f"cross_M{M}_{r}": Workload(f"cross_M{M}_{r}", M, 6144, 256, 8, 256, W_MXFP4, 2.5,
                                         "normal" if r == "spread" else r, False)
             for M in (1, 2, 4, 8, 12, 16) for r in ("spread", "hot")}


# Block-FP8 prefill sizes (the TP4 rank slice, Zipf routing): where the
# weights-on-M grouped GEMMs and the wide (pairs-on-M) ones cross over.
FP8_CROSSOVER = {f"fp8cross_M{M}": Workload(f"fp8cross_M{M}", M, 6144, 256, 8, 512, W_FP8_BLOCK128, 2.5, "zipf1.1",
                                            False)
                 for M in (512, 1024, 2048, 4096)}


# Reduced shapes for profiler captures that must hold only a few GB on the
# device: the block-FP8 prefill shape with 64 experts instead of 256.
PROFILE = {"prefill_fp8_e64": Workload("prefill_fp8_e64", 1024, 6144, 64, 8, 512, W_FP8_BLOCK128, 2.5, "zipf1.1", False)}


def _rng(seed: int, tag: str, *idx: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TAGS[tag], *idx])))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 draws to bf16 (nearest, ties to even) and return the bits."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


class Inputs:
    """Activations, router logits and a lazy per-expert weight source."""

    def __init__(self, wl: Workload, seed: int = 0):
        self.wl = wl
        self.seed = seed
        M, H, E = wl.M, wl.H, wl.E
        self.x = to_bf16_bits(_rng(seed, "x").standard_normal((M, H), dtype=np.float32))
        self.logits = self._logits()
        self.bias = (_rng(seed, "bias").standard_normal(E, dtype=np.float32) * np.float32(0.1)
                     if wl.bias else None)

    def _logits(self) -> np.ndarray:
        wl, seed = self.wl, self.seed
        M, E = wl.M, wl.E
        if wl.logits == "normal":
            return _rng(seed, "logits").standard_normal((M, E), dtype=np.float32)
        if wl.logits == "skew16":
            l = _rng(seed, "logits").standard_normal((M, E), dtype=np.float32)
            hot = _rng(seed, "hot").choice(E, size=min(16, E), replace=False)
            l[:, hot] += np.float32(2.0)
            return l
        if wl.logits in ("hot", "mixed"):
            # hot: every token prefers the same topk experts (N(0,1) + 6.0 on a
            # seeded set of topk experts), so few distinct experts are read;
            # mixed: the first half of the tokens hot, the rest spread N(0,1)
            l = _rng(seed, "logits").standard_normal((M, E), dtype=np.float32)
            hot = _rng(seed, "hotset").choice(E, size=min(wl.topk, E), replace=False)
            rows = slice(0, M) if wl.logits == "hot" else slice(0, (M + 1) // 2)
            l[rows, hot] += np.float32(6.0)
            return l
        if wl.logits.startswith("zipf"):
            a = float(wl.logits[4:])
            ranks = np.arange(1, E + 1, dtype=np.float64)
            p = ranks ** (-a)
            p /= p.sum()
            perm = _rng(seed, "perm").permutation(E)         # expert e has rank perm[e]
            g = _rng(seed, "gumbel").gumbel(size=(M, E))
            return (np.log(p[perm])[None, :] + g).astype(np.float32)
        raise ValueError(wl.logits)

    # weights are drawn per expert so large workloads never hold all fp32 copies
    def w13(self, e: int) -> np.ndarray:
        wl = self.wl
        return _rng(self.seed, "w13", e).standard_normal((2 * wl.I, wl.H), dtype=np.float32) * np.float32(0.02)

    def w2(self, e: int) -> np.ndarray:
        wl = self.wl
        return _rng(self.seed, "w2", e).standard_normal((wl.H, wl.I), dtype=np.float32) * np.float32(0.02)
