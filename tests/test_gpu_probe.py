"""The tensor-core probe (moe_probe_tensor_peak): measured MMA throughput per
kind, the denominator of the bench's tensor fraction.  On B200 the 8-bit kind
runs at twice the bf16 rate and the block-scaled 4-bit kind above the 8-bit
one; no kind exceeds the part's dense per-SM figure (8192 8-bit MACs per SM
clock)."""
import pytest

import prefill_moe_route_b200 as moe

pytestmark = pytest.mark.gpu


def test_tensor_probe_rates_are_consistent():
    fp8 = moe.moe_probe_tensor_peak(moe.MOE_PROBE_FP8, 4000)
    fp4 = moe.moe_probe_tensor_peak(moe.MOE_PROBE_FP4, 4000)
    bf16 = moe.moe_probe_tensor_peak(moe.MOE_PROBE_BF16, 4000)
    print("probe TFLOP/s, MAC/clk/SM:", {"fp8": fp8, "fp4": fp4, "bf16": bf16})
    for tf, mpc in (fp8, fp4, bf16):
        assert tf > 0 and mpc > 0
    assert 1.6 < fp8[1] / bf16[1] < 2.4
    assert fp4[1] > 1.2 * fp8[1]
    assert fp8[1] <= 8192 * 1.05 and fp4[1] <= 2 * 8192 * 1.05


def test_tensor_probe_is_repeatable():
    a = moe.moe_probe_tensor_peak(moe.MOE_PROBE_FP8, 2000)[1]
    b = moe.moe_probe_tensor_peak(moe.MOE_PROBE_FP8, 2000)[1]
    assert abs(a - b) / a < 0.05
