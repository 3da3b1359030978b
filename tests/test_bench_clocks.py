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


def test_profiled_traffic_only_for_the_captured_sources(monkeypatch):
    """A stored ncu traffic figure is reported only while the kernel sources
    hash to the value it was captured on; any edit turns it into None."""
    import hashlib
    import os
    files = ["csrc/decode_paged.cu", "csrc/sm100_ptx.cuh"]
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(bench.ROOT, "attention_flash_attn_02_b200", f), "rb") as fh:
            h.update(fh.read())
    current = h.hexdigest()[:16]
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "probe", {"files": files, "sha": current, "bytes": 1234})
    assert bench.profiled_traffic("probe") == 1234
    monkeypatch.setitem(bench.PROFILED_TRAFFIC, "probe", {"files": files, "sha": "0" * 16, "bytes": 1234})
    assert bench.profiled_traffic("probe") is None
