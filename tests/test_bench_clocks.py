"""bench.py's clock sampler on a fake NVML (no GPU): reason bits map to the names the timing
rules use, samples outside the timed window are dropped, the median clock is reported."""
import sys
import time
import types

import bench


def _fake_nvml(clocks, reasons):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    it = {"i": 0}
    m.nvmlInit = lambda: None
    m.nvmlDeviceGetHandleByPciBusId = lambda bus: ("bus", bus)
    m.nvmlDeviceGetHandleByIndex = lambda i: ("idx", i)
    m.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965

    def clock(h, c):
        it["i"] += 1
        return clocks[min(it["i"] - 1, len(clocks) - 1)]

    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetPowerUsage = lambda h: 512_000
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons[min(it["i"] - 1, len(reasons) - 1)]
    return m


def test_nvml_sampler(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965, 1800, 1965, 1965, 1965], [0, 0x4, 0x4 | 0x40, 0, 0]))
    c = bench.ClockSampler(0)
    t0 = time.time()
    c.start()
    time.sleep(0.2)
    c.stop()
    t1 = time.time()
    assert c.source == "nvml" and len(c.samples) >= 5
    s = c.summary(t0, t1)
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965 and s["power_w_max"] == 512.0
    assert s["reasons"] == ["hw_thermal_slowdown", "sw_power_cap"]
    assert s["samples"] == len(c.samples)
    # A window before every sample falls back to the last few samples rather than to nothing.
    assert c.summary(t0 - 10, t0 - 9)["samples"] == 5


def test_sampler_without_nvml_or_smi(monkeypatch):
    bad = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no driver")

    bad.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", bad)
    monkeypatch.setattr(bench.subprocess, "Popen", lambda *a, **k: (_ for _ in ()).throw(OSError("no nvidia-smi")))
    c = bench.ClockSampler(0)
    c.start()
    c.stop()
    assert c.source is None
    assert c.summary(0, time.time())["reasons"] == ["clock sampling unavailable"]
