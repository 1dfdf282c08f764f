"""GPU scenarios that need process-wide settings the library reads once per
process (MOE_FORCE_PATH, MOE_WAIT_TIMEOUT_MS, MOE_TEST_WITHHOLD_FLAG): the
tests run this file in a fresh child process with the variables set.

    python tests/gpu_child.py <mode> [json-args]

Prints one line per checked case and exits 0 when every check passed.
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import numpy as np  # noqa: E402
import torch  # noqa: E402

import prefill_moe_route_b200 as moe  # noqa: E402
from prefill_moe_route_b200.synth import Workload  # noqa: E402


def _wl(spec):
    return Workload(*spec)


def forced_large(specs):
    """Every workload runs on the grouped kernels and matches the oracle."""
    from test_gpu_parity import Problem
    assert os.environ.get("MOE_FORCE_PATH") == "large"
    for spec in specs:
        wl = _wl(spec)
        assert moe.moe_launches_per_call(wl.shape(), 0) > 1, wl.name
        pb = Problem(wl, seed=23)
        pb.check_weights()
        pb.run_and_check()
        print(f"ok forced-large {wl.name} M={wl.M}", flush=True)


def forced_small(specs):
    """Every workload runs on the single kernel (MOE_FORCE_PATH=small, where it
    would otherwise take the grouped kernels) and matches the oracle."""
    from test_gpu_parity import Problem
    assert os.environ.get("MOE_FORCE_PATH") == "small"
    for spec in specs:
        wl = _wl(spec)
        assert moe.moe_launches_per_call(wl.shape(), 0) == 1, wl.name
        pb = Problem(wl, seed=27)
        pb.run_and_check()
        print(f"ok forced-small {wl.name} M={wl.M}", flush=True)


def withhold(specs):
    """The first call leaves one mid flag unpublished: its waits run out, the
    call returns, the status reports the timeout and the wait site; the next
    call on the same workspace is normal again and matches the oracle."""
    from test_gpu_parity import Problem
    assert os.environ.get("MOE_TEST_WITHHOLD_FLAG") == "1"
    wl = _wl(specs[0])
    assert moe.moe_launches_per_call(wl.shape(), 0) == 1
    pb = Problem(wl, seed=29)
    pb.dev.forward()
    torch.cuda.synchronize()
    words = pb.dev.status_words()
    rc, st = pb.dev.status()
    site = int(words[2]) & 0xFFFFFFFF
    assert rc == moe.MOE_ERR_DEVICE_TIMEOUT, (rc, st)
    assert st & 1, st                                   # the timeout bit of the status word
    assert site >> 31 == 1 and ((site >> 24) & 0x7F) == 7, hex(site)   # recorded by the single-launch kernel
    print(f"ok timed out: status {st:#x}, first wait site {site:#x}", flush=True)
    rc, st = pb.dev.status()
    assert rc == moe.MOE_OK and st == 0                 # the query cleared it
    pb.run_and_check()
    print("ok next call matches the oracle", flush=True)


def static_withhold(specs):
    """The same through moe_forward_static: moe_get_status_static reports the
    timeout, and the next static call is bit-identical to moe_forward."""
    from harness_static import static_call
    from test_gpu_parity import Problem
    wl = _wl(specs[0])
    pb = Problem(wl, seed=31)
    got = static_call(pb.dev)
    rc, st = moe.moe_get_status_static()
    assert rc == moe.MOE_ERR_DEVICE_TIMEOUT and st & 1, (rc, st)
    print(f"ok static call timed out: status {st:#x}", flush=True)
    del got
    want, _ = pb.run_and_check()
    got = static_call(pb.dev)
    rc, st = moe.moe_get_status_static()
    assert rc == moe.MOE_OK and st == 0, (rc, st)
    assert np.array_equal(got, want)
    print("ok next static call is bit-identical to moe_forward", flush=True)


def static_forced_large(specs):
    """moe_forward_static on the grouped kernels: bit-identical to moe_forward."""
    from harness_static import static_call
    from test_gpu_parity import Problem
    assert os.environ.get("MOE_FORCE_PATH") == "large"
    for spec in specs:
        wl = _wl(spec)
        pb = Problem(wl, seed=37)
        want, _ = pb.run_and_check()
        for _ in range(2):
            got = static_call(pb.dev)
            rc, st = moe.moe_get_status_static()
            assert rc == moe.MOE_OK and st == 0, (rc, st)
            assert np.array_equal(got, want), wl.name
        print(f"ok static forced-large {wl.name}", flush=True)


MODES = {"forced_large": forced_large, "forced_small": forced_small, "withhold": withhold, "static_withhold": static_withhold,
         "static_forced_large": static_forced_large}

if __name__ == "__main__":
    MODES[sys.argv[1]](json.loads(sys.argv[2]) if len(sys.argv) > 2 else [])
    print("child ok", flush=True)
