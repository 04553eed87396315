"""bench.py's roofline denominator: the burst GEMM peak when the attention
kernel ran at full clock without a power cap (or in a short timed region),
the sustained one otherwise, and operations per clock per SM at the sampled
clock."""
import bench

PEAKS = {"bf16_tflops": 1635.2, "bf16_tflops_sustained": 1399.6}


def test_full_clock_uses_the_burst_peak():
    clk = {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": []}
    peak, note, kind = bench.roofline_peak(PEAKS, clk, 5000.0)
    assert kind == "burst" and peak == 2 * 1635.2 and "burst" in note


def test_power_cap_uses_the_sustained_peak():
    clk = {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    peak, _, kind = bench.roofline_peak(PEAKS, clk, 5000.0)
    assert kind == "sustained" and peak == 2 * 1399.6


def test_short_region_uses_the_burst_peak_and_no_file_the_fallback():
    clk = {"sm_mhz": 1400.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"]}
    assert bench.roofline_peak(PEAKS, clk, 200.0)[2] == "burst"
    assert bench.roofline_peak(None, clk, 200.0)[2] == "fallback"


def test_ops_per_clock_per_sm():
    # 16384 ops per clock per SM (the 8-bit MMA peak) at 1965 MHz on 148 SMs
    tops = 16384 * 1965e6 * 148 / 1e12
    assert abs(bench.ops_per_clk_per_sm(tops, 1965.0) - 16384) < 1e-6
    assert bench.ops_per_clk_per_sm(tops, None) is None
