"""Host logic of bench.py, on CPU: the clock sampler's summary (through a fake
NVML module, so no GPU is touched and no GPU setting is read or changed) and
the roofline bound of each workload shape."""
import os
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def fake_nvml(clocks, reasons):
    """A stand-in for pynvml that reports the given SM clocks and
    clock-event reason words in turn (the last one repeats)."""
    state = {"i": 0}
    m = types.SimpleNamespace()
    m.NVML_CLOCK_SM = 1
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetCount = lambda: 1
    m.nvmlDeviceGetHandleByIndex = lambda i: "h0"
    m.nvmlDeviceGetUUID = lambda h: "GPU-fake"
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        v = clocks[min(state["i"], len(clocks) - 1)]
        state["i"] += 1
        return v
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetPowerUsage = lambda h: 500_000
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[min(state["i"], len(reasons)) - 1]
    return m


def test_clock_sampler_summarises_fake_nvml(monkeypatch):
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml([1965, 1965, 1800, 1965], [0, 0x4, 0x4, 0]))
    cs = bench.ClockSampler("cpu", period_s=0.001)
    assert cs.nvml is not None
    cs.start()
    time.sleep(0.05)
    out = cs.stop()
    assert out["samples"] >= 4
    assert out["sm_max_mhz"] == 1965
    assert out["sm_mhz"] == 1965
    assert out["sm_min_mhz"] == 1800
    assert out["reasons"] == ["sw_power_cap"]
    assert out["source"].startswith("nvml")


def test_clock_sampler_flags_slowdown_reasons(monkeypatch):
    import bench
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml([1500], [0x8 | 0x40]))
    cs = bench.ClockSampler("cpu", period_s=0.001)
    cs.start()
    time.sleep(0.02)
    out = cs.stop()
    assert set(out["reasons"]) == {"hw_slowdown", "hw_thermal_slowdown"}


def test_default_workload_covers_the_five_configurations():
    import bench
    wl = bench.WORKLOADS["all"]
    assert wl["headline"] == "prefill"
    shapes = sum(len(bench.WORKLOADS[p]["shapes"]) * len(bench.WORKLOADS[p].get("M", [1]))
                 for p in wl["parts"])
    assert shapes == 1 + 3 + 2 + 2 + 12
