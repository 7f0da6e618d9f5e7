"""The benchmark's clock sampler on CPU, against a fake NVML module: it samples
during the region (the first sample before the region starts), reports the
median SM clock, the maximum, and every throttle reason seen in any sample, and
only reads (the fake has no setter, so a write would fail the test)."""
import sys
import time
import types

import bench


def fake_nvml(clocks, reasons):
    state = {"i": 0}
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: "h"
    m.nvmlDeviceGetHandleByIndex = lambda i: "h"
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        v = clocks[min(state["i"], len(clocks) - 1)]
        return v

    def why(h):
        v = reasons[min(state["i"], len(reasons) - 1)]
        state["i"] += 1
        return v

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = why
    return m


def sample(monkeypatch, clocks, reasons, seconds=0.05):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(clocks, reasons))
    with bench.ClockSampler(0) as clk:
        assert clk.samples, "no sample before the timed region"
        time.sleep(seconds)
    return clk.summary()


def test_samples_clock_and_reasons(monkeypatch):
    s = sample(monkeypatch, [1965, 1965, 1950, 1965], [0, 0x4, 0, 0x4 | 0x1])
    assert s["source"].startswith("nvml") and s["samples"] >= 2
    assert s["sm_max_mhz"] == 1965 and s["sm_mhz"] in (1950, 1965)
    assert s["reasons"] == ["sw_power_cap"]       # the idle bit is not a throttle reason


def test_thermal_and_hw_slowdown_are_reported(monkeypatch):
    s = sample(monkeypatch, [1400], [0x8, 0x40, 0x20])
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert s["sm_mhz"] == 1400


def test_short_region_still_has_a_sample(monkeypatch):
    s = sample(monkeypatch, [1965], [0], seconds=0.0)
    assert s is not None and s["samples"] >= 1
