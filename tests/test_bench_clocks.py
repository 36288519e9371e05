"""The bench's clock record, on the CPU against a fake NVML: the reader thread
samples while work runs, reports the median loaded SM clock and every
clock-event reason it saw, and nothing else."""
import sys
import time
import types

import bench


def _fake_nvml(clocks, reasons):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    state = {"i": 0}
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByUUID = lambda uuid: ("handle", uuid)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[state["i"] % len(clocks)]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return m


def _props(monkeypatch):
    import torch
    props = types.SimpleNamespace(uuid="12345678-0000-0000-0000-000000000000")
    monkeypatch.setattr(torch.cuda, "get_device_properties", lambda i: props)


def test_sampler_reports_clock_and_power_cap(monkeypatch):
    _props(monkeypatch)
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965.0, 1905.0, 1965.0], 0x4))
    s = bench.ClockSampler(0)
    time.sleep(0.05)
    r = s.stop()
    assert r["source"].startswith("nvml")
    assert r["samples"] >= 5
    assert r["sm_max_mhz"] == 1965.0
    assert r["sm_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_sampler_flags_thermal_slowdown_and_ignores_idle_samples(monkeypatch):
    _props(monkeypatch)
    # hw_thermal_slowdown (0x40) plus the idle bit (0x1), which is not reported
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1500.0, 300.0], 0x40 | 0x1))
    s = bench.ClockSampler(0)
    time.sleep(0.05)
    r = s.stop()
    assert r["reasons"] == ["hw_thermal_slowdown"]
    assert r["sm_mhz"] == 1500.0  # samples below 30% of max are idle, not load
