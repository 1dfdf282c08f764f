#!/usr/bin/env python3
"""µs per quantized routed-expert MoE call on B200, with roofline fractions.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload all|NAME] [--no-cpu-baseline] [--flush write|read|none]

A step is one whole MoE call (route -> align -> activation quant -> GEMM1 +
SwiGLU + mid quant -> GEMM2 -> combine) on one batch of synthetic inputs.
By default every workload runs, one JSON line each, in the order tiny,
decode_tp8, decode_tp4_skew, prefill_tp8 and last prefill_tp4_fp8 (M=4096,
block-FP8 experts: the largest one-GPU workload, the headline line).

Per workload: W warm-up steps, then exactly K timed steps (each a CUDA-graph
replay of one moe_forward, CUDA events around it, L2 flushed by a 256 MiB write
before it, outside the events) give `value`; then a larger sample of the same
replays gives the median / p10 / p90 spread, an L2-hot median, the per-kernel
device times and the end-to-end time through the C ABI with pinned host
buffers.  Bookends: a sample of every workload is timed before and after all
of the measurements and the drift between the two medians is reported.
With N > 1 (torchrun, one process per GPU) every rank runs independent
replicas on its own batches: there is no data-path collective.

--impl reference times the CPU oracle (oracle/) on the host cores instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "µs per MoE call and achieved fraction of HBM/tensor roofline"
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0
ORDER = ["tiny", "decode_tp8", "decode_tp4_skew", "prefill_tp8", "prefill_tp4_fp8"]
DRIFT_LIMIT = 0.03


def _all_workloads():
    from prefill_moe_route_b200.synth import CROSSOVER, FP8_CROSSOVER, MEDIUM, PROFILE, WORKLOADS
    return {**WORKLOADS, **MEDIUM, **CROSSOVER, **FP8_CROSSOVER, **PROFILE}


def _args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="all",
                   choices=["all", "medium", "crossover", "fp8crossover"] + list(_all_workloads()),
                   help="all: the five workloads (default); medium: M = 32..512 under spread/hot/mixed routing; "
                        "crossover: decode sizes M = 1..16 (run once with MOE_FORCE_PATH=small, once with =large); "
                        "fp8crossover: block-FP8 prefill sizes M = 512..4096")
    p.add_argument("--profile-calls", type=int, default=0,
                   help="only run this many eager calls of each workload (for a profiler) and print nothing")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=8.0)
    p.add_argument("--flush", choices=["write", "read", "none"], default="write",
                   help="L2 between timed steps: write a 256 MiB buffer (default), read it, or keep it hot")
    return p.parse_args(argv)


def _workloads(name):
    from prefill_moe_route_b200.synth import CROSSOVER, FP8_CROSSOVER, MEDIUM
    if name == "all":
        return list(ORDER)
    if name == "medium":
        return list(MEDIUM)
    if name == "crossover":
        return list(CROSSOVER)
    if name == "fp8crossover":
        return list(FP8_CROSSOVER)
    return [name]


def _spread_samples(wl, steps):
    """Samples for the spread and the bookends: >= 100 (>= 30 at M >= 4096)."""
    return max(steps, 30 if wl.M >= 4096 else 100)


def _workload_config(wl):
    fmt = "mxfp4" if wl.wfmt == 1 else "fp8_block128"
    return {"workload": f"{wl.name} (M={wl.M}, H={wl.H}, E={wl.E}, top-{wl.topk}, I={wl.I}, {fmt} experts, "
                        f"routed scale {wl.routed_scale})",
            "M": wl.M, "H": wl.H, "E": wl.E, "topk": wl.topk, "I": wl.I, "weights": fmt,
            "router_logits": wl.logits, "l2": "flushed before every timed step (256 MiB write, outside the events)",
            "timing": "each step a CUDA-graph replay of one moe_forward, CUDA events around it"}


# DRAM traffic per launch (ncu dram__bytes_read.sum + dram__bytes_write.sum,
# one capture of the full-size workload; profiles/ has the summaries), valid
# only for the sources it was measured on: each kernel is keyed by the sha256
# of the files that define it and its launch plan (its .cu file, api.cu and
# the shared headers).  Any change to them reports null.
_GEMM_SRC = ("gemm.cu", "api.cu", "ptx.cuh", "codec.cuh", "internal.h")
_SMALL_SRC = ("small.cu", "api.cu", "ptx.cuh", "codec.cuh", "internal.h")
_GEMM_MEASURED = "0ec4d77386dc7a893e65cf0b22844d368b620a655d5decc5a815f7d8cbe26e1d"
_SMALL_MEASURED = "a63117e641e5c63569e41f63fff806cd201d72692028d6407ada9c23764fd55b"
_NCU_TRAFFIC = {
    "decode_tp8": {"moe_small": (_SMALL_SRC, _SMALL_MEASURED, 73127424 + 1673216)},
    "prefill_tp8": {"gemm1": (_GEMM_SRC, _GEMM_MEASURED, 459781120 + 4726784),
                    "gemm2": (_GEMM_SRC, _GEMM_MEASURED, 216362752 + 69238784)},
    "prefill_tp4_fp8": {"gemm1": (_GEMM_SRC, _GEMM_MEASURED, 1877602304 + 22433792),
                        "gemm2": (_GEMM_SRC, _GEMM_MEASURED, 823742464 + 383138048)},
}


def _kernel_source_hash(files) -> str:
    import hashlib
    csrc = os.path.join(ROOT, "prefill_moe_route_b200", "csrc")
    h = hashlib.sha256()
    for name in sorted(files):
        h.update(name.encode())
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(f.read())
    with open(os.path.join(ROOT, "include", "moe_b200.h"), "rb") as f:
        h.update(f.read())
    return h.hexdigest()


def _traffic(workload: str, kernel: str):
    entry = _NCU_TRAFFIC.get(workload, {}).get(kernel)
    if entry is None:
        return None
    files, measured, nbytes = entry
    return nbytes if _kernel_source_hash(files) == measured else None


def _l2_note(mode):
    return {"write": "flushed before every timed step (256 MiB write, outside the events)",
            "read": "flushed before every timed step (256 MiB read, outside the events)",
            "none": "hot: no flush between steps"}[mode]


def _dtype(wl):
    return "e2m1 x e2m1 (mxfp4), e4m3 mid, fp32 accumulate" if wl.wfmt == 1 else "e4m3 x e4m3, fp32 accumulate"


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _probe_peaks():
    """The tensor cores' measured rates on this GPU (moe_probe_tensor_peak):
    {"fp8": TFLOP/s, "fp4": TFLOP/s, ...}, or None when the probe fails."""
    import prefill_moe_route_b200 as moe
    try:
        out = {}
        for name, kind in (("fp8", moe.MOE_PROBE_FP8), ("fp4", moe.MOE_PROBE_FP4), ("bf16", moe.MOE_PROBE_BF16)):
            tf, mpc = moe.moe_probe_tensor_peak(kind, 4000)
            out[name] = round(tf, 1)
            out[name + "_mac_per_clk_sm"] = round(mpc, 1)
        return out
    except Exception as e:  # the fraction then uses the bf16-derived rates
        print(f"tensor probe unavailable: {e}", file=sys.stderr)
        return None


def _tensor_context(wl, value_us: float, probe=None):
    """The tensor-core side of the roofline, for context: the call's
    algorithmic FLOPs 2*M*k*(2I*H + H*I) over the rate of the MMA kind each
    GEMM issues -- measured by the library's probe (MXFP4 GEMM1: kind::mxf4;
    block-FP8 GEMMs and MXFP4 GEMM2: the 8-bit kind), else derived from the
    measured bf16 GEMM peak (x4 for E2M1 x E2M1, x2 for 8-bit operands) -- as a
    time floor and its fraction of the call."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            bf16, kind = float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        bf16, kind = FALLBACK_BF16_TFLOPS, "fallback"
    P = wl.M * wl.topk
    f1, f2 = 2.0 * P * 2 * wl.I * wl.H, 2.0 * P * wl.H * wl.I
    r1, r2 = (4.0, 2.0) if wl.wfmt == 1 else (2.0, 2.0)   # GEMM1, GEMM2 rate over bf16
    out = {"flops": f1 + f2, "achieved_tflops": (f1 + f2) / (value_us * 1e-6) / 1e12}
    derived_us = (f1 / (bf16 * r1) + f2 / (bf16 * r2)) * 1e-6
    if probe:
        p1 = probe["fp4"] if wl.wfmt == 1 else probe["fp8"]
        t_floor_us = (f1 / p1 + f2 / probe["fp8"]) * 1e-6
        out.update({"t_floor_us": t_floor_us, "frac": t_floor_us / value_us,
                    "peak_basis": f"measured by the library's tcgen05 probe: GEMM1 {p1} TFLOP/s "
                                  f"({'kind::mxf4' if wl.wfmt == 1 else 'kind::f8f6f4'}), GEMM2 {probe['fp8']} "
                                  f"TFLOP/s (kind::f8f6f4)",
                    "probe": probe,
                    "frac_vs_bf16_derived": derived_us / value_us})
    else:
        out.update({"t_floor_us": derived_us, "frac": derived_us / value_us,
                    "peak_basis": f"{kind} bf16 {bf16} TFLOP/s x {r1:g} (GEMM1) / x {r2:g} (GEMM2)"})
    return out


def unit_bytes(wl):
    """Algorithmic bytes of one selected expert: (w13 payload + scales, w2 payload + scales)."""
    H, I = wl.H, wl.I
    if wl.wfmt == 1:
        return 2 * I * H // 2 + 2 * I * H // 32, H * I // 2 + H * I // 32
    return 2 * I * H + (2 * I // 128) * (H // 128) * 4, H * I + (H // 128) * (I // 128) * 4


def algorithmic_bytes(wl, ndist: float):
    """Per kernel and per call: selected experts' weights + activations the step reads or writes."""
    H, M, P = wl.H, wl.M, wl.M * wl.topk
    w13_unit, w2_unit = unit_bytes(wl)
    act1 = M * (H // 2 + H // 32) if wl.wfmt == 1 else M * (H + H // 128 * 4)
    mid_bytes = P * (wl.I + wl.I // 128 * 4)
    call = ndist * (w13_unit + w2_unit) + M * H * 2 + M * wl.E * 4 + M * H * 2
    return {"gemm1": ndist * w13_unit + act1 + mid_bytes,
            "gemm2": ndist * w2_unit + mid_bytes + P * H * 4,
            "moe_small": call + mid_bytes,
            "call": call}


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """Polls SM clock and clock-event reasons through NVML (about every ms) while it is open."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.001)

    def __enter__(self):
        if self._nv is not None:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": sorted(self.reasons - {"gpu_idle"})}


# --------------------------------------------------------------------- oracle timing
class OracleSample:
    """The oracle on a bounded token sample of one workload: the experts those
    tokens route to are quantized once by the oracle's own codecs; every run
    is one oracle forward over the sample."""

    def __init__(self, wl, flops_budget: float = 1.5e9):
        import numpy as np

        import oracle
        from prefill_moe_route_b200.synth import Inputs
        self.wl = wl
        inputs = Inputs(wl, seed=0)
        per_token_flops = 2 * wl.topk * (2 * wl.I * wl.H + wl.H * wl.I)
        self.n = int(max(1, min(wl.M, flops_budget // per_token_flops)))
        self.tokens = np.arange(self.n, dtype=np.int32)
        self.ids, self.tw = oracle.route(inputs.logits, inputs.bias, wl.topk, wl.routed_scale)
        E, H, I = wl.E, wl.H, wl.I
        if wl.wfmt == 1:
            arr = [np.zeros((E, 2 * I, H // 2), np.uint8), np.zeros((E, 2 * I, H // 32), np.uint8),
                   np.zeros((E, H, I // 2), np.uint8), np.zeros((E, H, I // 32), np.uint8)]
        else:
            arr = [np.zeros((E, 2 * I, H), np.uint8), np.ones((E, 2 * I // 128, H // 128), np.float32),
                   np.zeros((E, H, I), np.uint8), np.ones((E, H // 128, I // 128), np.float32)]
        for e in sorted(set(self.ids[self.tokens].reshape(-1).tolist())):
            if wl.wfmt == 1:
                q = (*oracle.quant_mxfp4(inputs.w13(e)), *oracle.quant_mxfp4(inputs.w2(e)))
            else:
                q = (*oracle.quant_fp8_block128(inputs.w13(e)), *oracle.quant_fp8_block128(inputs.w2(e)))
            for a, v in zip(arr, q):
                a[e] = v
        self.x = inputs.x
        self.arr = arr

    def run_once(self) -> float:
        """One oracle forward over the sample; returns µs per whole call (scaled by M / n)."""
        import oracle
        t0 = time.perf_counter()
        oracle.forward_tokens(self.wl.shape(), self.x, self.ids, self.tw, *self.arr, tokens=self.tokens,
                              want_midq=False)
        return (time.perf_counter() - t0) * 1e6 * (self.wl.M / self.n)

    def timed(self, seconds: float, threads: int | None = None):
        """Runs for about `seconds` (at least once); returns (µs per call, runs, threads used)."""
        import oracle
        prev = oracle.set_threads(threads) if threads else None
        try:
            used = oracle.set_threads(0)
            runs, t_us, t0 = 0, 0.0, time.perf_counter()
            while True:
                t_us += self.run_once()
                runs += 1
                if time.perf_counter() - t0 >= seconds:
                    break
            return t_us / runs, runs, used
        finally:
            if prev:
                oracle.set_threads(prev)


def time_oracle(wl, seconds: float, max_runs: int | None = None):
    """Oracle forward on a bounded token sample; returns (µs per whole call, runs, tokens, threads)."""
    s = OracleSample(wl)
    us, runs, used = s.timed(seconds if max_runs is None else 0.0)
    return us, runs, s.n, used


# --------------------------------------------------------------------- reference arm
def max_over_ranks(v: float, dist=None, device="cpu") -> float:
    """The largest of every rank's `v` (all ranks call it; identity without a process group)."""
    if dist is None:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_us_per_call(local_ms_per_call: float, world: int, dist=None, device="cpu"):
    """(slowest rank's ms per call, whole-job us per call): N replicas each run
    one call per step, so the job finishes N calls in the slowest rank's step."""
    step_ms = max_over_ranks(local_ms_per_call, dist, device)
    return step_ms, step_ms * 1000.0 / world


def _value_kind(world: int) -> str:
    if world == 1:
        return "device µs per call (mean of the timed steps)"
    return (f"job µs per call over {world} replicas: the slowest rank's mean step time / {world} "
            f"(a replica-throughput figure, not one call's latency)")


def run_reference(args):
    WORKLOADS = _all_workloads()
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for name in _workloads(args.workload):
        wl = WORKLOADS[name]
        sample = OracleSample(wl, flops_budget=0.4e9)
        per_step = []
        for i in range(args.warmup + args.steps):   # one bounded oracle sample per step
            us = sample.run_once()
            if i >= args.warmup:
                per_step.append(us)
        import oracle
        threads = oracle.set_threads(0)
        v = statistics.mean(per_step)
        desc = f"{sample.n} of {wl.M} tokens per step, scaled to a whole call"
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "us", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": v / 1000.0, "higher_is_better": False,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64 (oracle)", "data": "synthetic",
                "config": dict(_workload_config(wl), l2="host run: not applicable",
                               timing="each step one bounded oracle sample on the host cores, wall clock"),
                "cpu_baseline": {"value": v, "unit": "us", "cores": threads, "kind": "oracle", "sample": desc},
                "e2e": {"value": v, "unit": "us", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)


# --------------------------------------------------------------------- our arm
class Case:
    """One workload on this rank's GPU: weights, input sets and the CUDA graphs that replay the call."""

    def __init__(self, wl, rank: int, local: int, flush):
        import numpy as np
        import torch

        import prefill_moe_route_b200 as moe
        from prefill_moe_route_b200.harness import DeviceMoE
        from prefill_moe_route_b200.synth import Inputs

        self.wl, self.flush = wl, flush
        self.stream = torch.cuda.current_stream()
        self.dev = DeviceMoE(wl, Inputs(wl, seed=0), device=f"cuda:{local}")
        dev = self.dev
        self.nsets = 4 if wl.M >= 1024 else 16
        self.acts = [Inputs(wl, seed=1 + 100000 * rank + i) for i in range(self.nsets)]
        self.X = [torch.from_numpy(a.x.view(np.int16)).cuda() for a in self.acts]
        self.L = [torch.from_numpy(a.logits).cuda() for a in self.acts]
        self.launches = moe.moe_launches_per_call(wl.shape(), torch.cuda.current_device())

        def made_event():
            e = torch.cuda.Event(enable_timing=True)
            e.record(self.stream)         # torch creates the CUDA event on first record
            return e

        self.kev = [[made_event() for _ in range(5)] for _ in range(self.nsets)]
        for i in range(self.nsets):      # eager warm-up outside capture (one-time set-up of the library)
            dev.forward(x=self.X[i], logits=self.L[i])
        torch.cuda.synchronize()
        self.graphs, self.kgraphs = [], []
        for i in range(self.nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                dev.forward(x=self.X[i], logits=self.L[i])
            self.graphs.append(g)
            kg = torch.cuda.CUDAGraph()
            with torch.cuda.graph(kg):
                moe.moe_forward_timed(dev.shape, self.X[i], self.L[i], dev.bias, dev.w13, dev.sf13, dev.w2,
                                      dev.sf2, dev.out, dev.workspace, dev.ws_bytes, self.kev[i])
            self.kgraphs.append(kg)
        torch.cuda.synchronize()

    def replay_timed(self, n: int, start: int = 0, flush: bool = True):
        """n replays, each bracketed by CUDA events (L2 flushed before each unless flush=False); ms each."""
        import torch
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
        for i in range(n):
            if flush:
                self.flush()
            ev[i][0].record(self.stream)
            self.graphs[(start + i) % self.nsets].replay()
            ev[i][1].record(self.stream)
        torch.cuda.synchronize()
        return [a.elapsed_time(b) for a, b in ev]

    def kernel_times(self, n: int):
        """Per-kernel device ms (events between the launches) and the mean count of selected experts."""
        import numpy as np
        import torch
        names = ["route", "gemm1", "gemm2", "combine"]
        kt = {k: [] for k in names}
        distinct, wl, dev = [], self.wl, self.dev
        for i in range(n):
            self.flush()
            self.kgraphs[i % self.nsets].replay()
            torch.cuda.synchronize()
            evs = self.kev[i % self.nsets]
            for j, k in enumerate(names):
                kt[k].append(evs[j].elapsed_time(evs[j + 1]))
            counts = dev.workspace[dev.layout["counts"]:dev.layout["counts"] + 4 * wl.E].cpu().numpy().view(np.int32)
            distinct.append(int((counts > 0).sum()))
        return {k: statistics.mean(v) for k, v in kt.items()}, statistics.mean(distinct)

    def e2e(self, warmup: int, steps: int, world: int, dist):
        """The same call end to end: x and logits copied in from one pinned host buffer, the call,
        out copied back, every step (captured once per input set as a decode loop would run it)."""
        import numpy as np
        import torch
        dev, X, L = self.dev, self.X, self.L
        xb, lb = X[0].numel() * 2, L[0].numel() * 4
        hxl = []
        for a in self.acts:
            buf = torch.empty(xb + lb, dtype=torch.uint8).pin_memory()
            buf[:xb].copy_(torch.from_numpy(a.x.view(np.uint8).reshape(-1)))
            buf[xb:].copy_(torch.from_numpy(a.logits.view(np.uint8).reshape(-1)))
            hxl.append(buf)
        dxl = torch.empty(xb + lb, dtype=torch.uint8, device="cuda")
        dx, dl = dxl[:xb].view(torch.int16).view(X[0].shape), dxl[xb:].view(torch.float32).view(L[0].shape)
        hout = torch.empty(dev.out.shape, dtype=dev.out.dtype).pin_memory()

        def e2e_step(i):
            dxl.copy_(hxl[i % self.nsets], non_blocking=True)
            dev.forward(x=dx, logits=dl)
            hout.copy_(dev.out, non_blocking=True)

        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            e2e_step(0)   # warms the call cache outside the capture
        torch.cuda.current_stream().wait_stream(side)
        egraphs = []
        for i in range(self.nsets):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                e2e_step(i)
            egraphs.append(g)
        for i in range(warmup):
            egraphs[i % self.nsets].replay()
        torch.cuda.synchronize()
        ee = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for i in range(steps):
            self.flush()
            ee[i][0].record(self.stream)
            egraphs[i % self.nsets].replay()
            ee[i][1].record(self.stream)
        torch.cuda.synchronize()
        e2e_us = whole_job_us_per_call(statistics.mean([a.elapsed_time(b) for a, b in ee]), world, dist, "cuda")[1]
        if not np.array_equal(hout.numpy().view(np.uint16), dev.out.cpu().numpy().view(np.uint16)):
            raise SystemExit("end-to-end result read back differs from the device output")
        del egraphs
        h2d = X[0].numel() * 2 + L[0].numel() * 4
        d2h = dev.out.numel() * 2
        return {"value": e2e_us, "unit": "us", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}


def _spread(t_ms):
    qs = statistics.quantiles(t_ms, n=10) if len(t_ms) >= 2 else [t_ms[0]] * 9
    return {"median_us": statistics.median(t_ms) * 1000.0, "p10_us": qs[0] * 1000.0, "p90_us": qs[-1] * 1000.0,
            "samples": len(t_ms)}


def run_ours(args):
    import torch

    import prefill_moe_route_b200 as moe
    WORKLOADS = _all_workloads()

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    moe.load()
    flush_buf = torch.zeros(256 << 20, dtype=torch.uint8, device="cuda")
    flush_sink = torch.zeros(1, dtype=torch.int64, device="cuda")

    def flush():
        if args.flush == "write":
            flush_buf.zero_()
        elif args.flush == "read":
            torch.sum(flush_buf.view(torch.int64), 0, keepdim=True, out=flush_sink)

    names = _workloads(args.workload)
    if args.profile_calls:
        # a profiler's run: the same set-up, then a few eager calls per workload, no timing
        from prefill_moe_route_b200.harness import DeviceMoE
        from prefill_moe_route_b200.synth import Inputs
        for n in names:
            dev = DeviceMoE(WORKLOADS[n], Inputs(WORKLOADS[n], seed=0), device=f"cuda:{local}")
            for _ in range(args.profile_calls):
                flush()
                dev.forward()
            torch.cuda.synchronize()
            rc, st = dev.status()
            if rc != moe.MOE_OK:
                raise SystemExit(f"{n}: device status {st}")
            del dev
        return
    cases = {n: Case(WORKLOADS[n], rank, local, flush) for n in names}
    peak, peak_kind = _peaks()
    probe = _probe_peaks()   # the tensor cores' measured rates on this GPU (~3 ms)

    # bookends: a sample of every workload before and after all measurements
    def bookend():
        out = {}
        for n in names:
            c = cases[n]
            c.replay_timed(3, flush=args.flush != "none")
            out[n] = statistics.median(c.replay_timed(_spread_samples(c.wl, 0) // 2, flush=args.flush != "none"))
        return out

    with ClockSampler(local) as clk_all:
        before = bookend()
        results = {}
        for n in names:
            c, wl = cases[n], cases[n].wl
            with ClockSampler(local) as clk:
                # ---- the timed steps: exactly K, bracketed by barrier + synchronize, max over ranks
                c.replay_timed(args.warmup, flush=args.flush != "none")
                barrier()
                t_ms = c.replay_timed(args.steps, start=args.warmup, flush=args.flush != "none")
                barrier()
                rc, st = c.dev.status()
                if rc != moe.MOE_OK:
                    raise SystemExit(f"{n}: device status {st} after the timed steps")
                step_ms, value_us = whole_job_us_per_call(statistics.mean(t_ms), world, dist, "cuda")
                spread = _spread(c.replay_timed(_spread_samples(wl, args.steps), flush=args.flush != "none"))
                hot = _spread(c.replay_timed(_spread_samples(wl, args.steps), flush=False))
                kmean, ndist = c.kernel_times(min(args.steps, 20))
                e2e = c.e2e(args.warmup, args.steps, world, dist)
            results[n] = dict(t_ms=t_ms, step_ms=step_ms, value_us=value_us, spread=spread, hot=hot, kmean=kmean,
                              ndist=ndist, e2e=e2e, clocks=clk.summary())
        after = bookend()

    for n in names:
        c, wl, r = cases[n], cases[n].wl, results[n]
        alg = algorithmic_bytes(wl, r["ndist"])
        kmean = r["kmean"]
        if c.launches == 1:   # the decode-sized path runs the whole call as one kernel (events 1..4 follow it)
            kms = {"moe_small": kmean["route"]}
            dom = "moe_small"
        else:
            kms = dict(kmean)
            dom = max(("gemm1", "gemm2"), key=lambda k: kmean[k])
        w13_unit, w2_unit = unit_bytes(wl)
        achieved = alg[dom] / (kms[dom] * 1e-3) / 1e9
        roofline = {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "peak_kind": f"hbm copy GB/s, {peak_kind}",
                    "traffic": _traffic(wl.name, dom),
                    "algorithmic_bytes_per_launch": alg[dom],
                    "unit_bytes": {"moe_small": w13_unit + w2_unit, "gemm1": w13_unit, "gemm2": w2_unit}[dom],
                    "units_per_launch": r["ndist"],
                    "kernel_ms": kms,
                    "whole_call": {"algorithmic_bytes": alg["call"],
                                   "frac_of_hbm_at_value": alg["call"] / (r["value_us"] * 1e-6) / 1e9 / peak},
                    "tensor": _tensor_context(wl, r["value_us"], probe)}
        drift = abs(after[n] - before[n]) / before[n]
        cpu = None
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            sample = OracleSample(wl)
            us, runs, threads = sample.timed(args.cpu_seconds)
            us1, runs1, _ = sample.timed(args.cpu_seconds / 2, threads=1)
            cpu = {"value": us, "unit": "us", "cores": threads, "kind": "oracle",
                   "sample": f"{runs} oracle runs over {sample.n} of {wl.M} tokens of one {wl.name} batch, "
                             f"scaled to a whole call",
                   "one_core": {"value": us1, "unit": "us", "cores": 1, "runs": runs1}}
        if rank == 0:
            line = {"metric": METRIC, "value": r["value_us"], "unit": "us", "n_gpus": world, "steps": args.steps,
                    "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": False, "scaling": "weak",
                    "vs_baseline": None, "dtype": _dtype(wl), "data": "synthetic",
                    "config": dict(_workload_config(wl), l2=_l2_note(args.flush)),
                    "roofline": roofline, "cpu_baseline": cpu, "e2e": r["e2e"],
                    "gpu_launches": c.launches * args.steps, "launches_per_call": c.launches,
                    "clocks": r["clocks"], "step_spread": r["spread"], "hot_l2": r["hot"],
                    "bookends": {"before_median_us": before[n] * 1000.0, "after_median_us": after[n] * 1000.0,
                                 "drift": drift, "within_limit": drift <= DRIFT_LIMIT, "limit": DRIFT_LIMIT},
                    "value_kind": _value_kind(world),
                    "path": "single kernel" if c.launches == 1 else "grouped kernels",
                    "parallelism": f"replicas x{world}" if world > 1 else "1 GPU"}
            print(json.dumps(line), flush=True)
    if rank == 0:
        print(json.dumps({"clocks_whole_run": clk_all.summary()}), file=sys.stderr, flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = _args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
