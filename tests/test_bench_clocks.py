"""bench.py's clock record, driven by a fake NVML on the CPU: the median SM
clock under load, the maximum clock, and every throttle reason seen during the
timed region (the bits NVML defines for them), without touching a GPU."""
import os
import sys
import types

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _fake_nvml(clocks, reason_bits):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    state = {"i": 0}
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda uuid: ("handle", uuid)
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        v = clocks[min(state["i"], len(clocks) - 1)]
        return v

    def reasons(h):
        b = reason_bits[min(state["i"], len(reason_bits) - 1)]
        state["i"] += 1
        return b

    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = reasons
    return nv


@pytest.fixture
def bench_with_fake_nvml(monkeypatch):
    def make(clocks, bits):
        monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(clocks, bits))
        props = types.SimpleNamespace(uuid="0000-fake")
        monkeypatch.setattr(torch.cuda, "get_device_properties", lambda d: props)
        import bench
        return bench
    return make


def test_clock_record_reports_median_max_and_reasons(bench_with_fake_nvml):
    bench = bench_with_fake_nvml([1900, 1950, 1300, 1965, 1920], [0x0, 0x4, 0x4 | 0x8, 0x0, 0x40])
    c = bench.Clocks(0)
    assert c.ok
    for _ in range(5):
        c._sample()
    s = c.summary()
    assert s["sm_mhz"] == 1920 and s["sm_max_mhz"] == 1965 and s["samples"] == 5
    assert s["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]


def test_clock_record_without_nvml_says_why(monkeypatch):
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("NVML not available")

    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    import bench
    c = bench.Clocks(0)
    assert not c.ok
    s = c.summary()
    assert s["sm_mhz"] is None and s["reasons"] == [] and "NVML" in s["error"]
