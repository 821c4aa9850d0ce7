"""Host logic of the benchmark line that needs no GPU: the clock-sample summary (including timed regions shorter
than the sampling period) and the MUFU roofline constants."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def row(ts, sm, mx=1965, power=500.0, cap="Not Active", uuid="GPU-abc"):
    # fields: timestamp, uuid, clocks.sm, clocks.max.sm, power.draw, active reasons, hw, hw_thermal, sw_thermal, sw_cap
    return (ts, ["2026/01/01", uuid, "%d MHz" % sm, "%d MHz" % mx, "%.1f W" % power, "0x0", "Not Active",
                 "Not Active", "Not Active", cap])


def test_summary_inside_the_timed_region():
    s = bench.ClockSampler("GPU-abc")
    s.rows = [row(0.9, 1000), row(1.0, 1800), row(1.1, 1700, cap="Active"), row(1.2, 1900), row(2.0, 500)]
    out = s.summary(1.0, 1.2)
    assert out["samples"] == 3 and out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"] and out["window"] == "timed region"
    assert out["power_w_max"] == 500.0


def test_summary_short_region_takes_the_neighbouring_samples():
    s = bench.ClockSampler("GPU-abc")
    s.rows = [row(0.5, 1000), row(0.9, 1600), row(1.3, 1700), row(2.0, 100)]
    out = s.summary(1.0, 1.01)  # no sample within [1.0, 1.16]
    assert out["samples"] == 2 and out["sm_mhz"] == 1650
    assert out["window"].startswith("nearest samples")


def test_summary_ignores_other_gpus_and_empty():
    s = bench.ClockSampler("GPU-abc")
    s.rows = [row(1.0, 1800, uuid="GPU-other")]
    assert s.summary(0.9, 1.1) is None
    s.rows = []
    assert s.summary(0.0, 1.0) is None


def test_mufu_bound_constants():
    # 16 exponentials per cycle per SM on 148 SMs at 1965 MHz, in TFLOP/s-equivalent for the forward at D = 64
    # (4 * 64 FLOP per exponential) and D = 128: the bound is below the tensor peak at D = 64 only.
    exp_per_s = bench.MUFU_EXP_PER_CYCLE_SM * bench.N_SMS * bench.NOMINAL_SM_MHZ * 1e6
    assert abs(exp_per_s * 256 / 1e12 - 1191.1) < 1.0
    assert exp_per_s * 256 / 1e12 < bench.FALLBACK_PEAKS["bf16_tflops"] < exp_per_s * 512 / 1e12
