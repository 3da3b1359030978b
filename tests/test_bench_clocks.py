"""The bench's clock sampler, on the CPU against a fake NVML module: samples
inside the timed region only, throttle reasons decoded from the bit mask."""
import sys
import time
import types

import bench


def _fake_nvml(reason_bits):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetCount = lambda: 2
    m.nvmlDeviceGetHandleByIndex = lambda i: i
    m.nvmlDeviceGetUUID = lambda h: f"GPU-0000-{h}"
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    m.nvmlDeviceGetClockInfo = lambda h, c: 1800 + h
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reason_bits
    return m


def test_nvml_sampler_reports_region_samples_and_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(0x4 | 0x1))
    c = bench.ClockSampler("0000-1", 0)   # matches device 1 by UUID
    c.start()
    time.sleep(0.03)                      # samples before the region are dropped
    c.begin()
    time.sleep(0.06)
    c.end()
    time.sleep(0.03)
    out = c.stop()
    assert out["source"].startswith("nvml")
    assert out["samples"] >= 3
    assert out["sm_mhz"] == 1801 and out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    inside = [r for r in c.rows if c.t0 <= r[0] <= c.t1]
    assert len(inside) == out["samples"] < len(c.rows)


def test_nvml_sampler_flags_thermal_slowdown(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(0x40 | 0x20))
    c = bench.ClockSampler("", 1)
    c.start()
    c.begin()
    time.sleep(0.03)
    c.end()
    out = c.stop()
    assert out["reasons"] == ["hw_thermal_slowdown", "sw_thermal_slowdown"]
