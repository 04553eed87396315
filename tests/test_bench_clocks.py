"""bench.py's clock sampler on a stand-in NVML (no GPU): samples are taken
from the start of the timed region, the median clock and the reasons the
bit masks name are reported, and a sampler without NVML falls back."""
import time

import bench


class FakeNVML:
    NVML_CLOCK_SM = 1

    def __init__(self, clocks, bits):
        self.clocks, self.bits, self.i, self.inits, self.shutdowns = clocks, bits, 0, 0, 0

    def nvmlInit(self):
        self.inits += 1

    def nvmlShutdown(self):
        self.shutdowns += 1

    def nvmlDeviceGetHandleByUUID(self, uuid):
        raise RuntimeError("no torch device here")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("dev", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        assert kind == self.NVML_CLOCK_SM
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        c = self.clocks[self.i % len(self.clocks)]
        self.i += 1
        return c

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.bits


def test_nvml_sampler_reports_median_and_reasons():
    nv = FakeNVML([1965, 1950, 1965, 1965, 1900], 0x4 | 0x1)
    with bench.ClockSampler(0, period_s=0.001, nvml=nv) as clk:
        time.sleep(0.02)
    out = clk.summary()
    assert out["source"] == "nvml" and out["samples"] >= 2
    assert out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] == 1965  # the pattern repeats: 3 of every 5 samples read 1965
    assert out["reasons"] == ["sw_power_cap"]  # idle (0x1) is not a reported reason
    assert nv.inits == 1 and nv.shutdowns == 1


def test_nvml_sampler_flags_thermal_and_hw_slowdown():
    nv = FakeNVML([1200], 0x8 | 0x40 | 0x20)
    with bench.ClockSampler(0, period_s=0.001, nvml=nv) as clk:
        pass
    out = clk.summary()
    assert out["samples"] >= 1  # a region shorter than the period still gets a sample
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_failing_nvml_falls_back():
    class Broken(FakeNVML):
        def nvmlInit(self):
            raise RuntimeError("no driver")

    clk = bench.ClockSampler(0, nvml=Broken([0], 0))
    assert not clk._start_nvml()
    assert clk.summary()["reasons"] == ["unsampled"]
