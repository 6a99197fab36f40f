"""bench.py's clock sampler against a fake NVML (no GPU): it keeps only the samples taken
inside the timed window, reports the median SM clock and every clock-event reason seen
there, and says "unsampled" when the window holds none (instead of idle clocks)."""
import sys
import time
import types

import bench


def _fake_nvml(mhz_seq, reasons_bits):
    calls = {"n": 0}
    mod = types.ModuleType("pynvml")
    mod.NVML_CLOCK_SM = 1

    def clock(h, kind):
        calls["n"] += 1
        return mhz_seq[min(calls["n"] - 1, len(mhz_seq) - 1)]

    mod.nvmlInit = lambda: None
    mod.nvmlDeviceGetHandleByPciBusId = lambda bus: ("handle", bus)
    mod.nvmlDeviceGetHandleByIndex = lambda i: ("handle", i)
    mod.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965
    mod.nvmlDeviceGetClockInfo = clock
    mod.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons_bits
    return mod


def test_window_median_and_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1700, 1710, 1720] * 1000, 0x4))
    c = bench.ClockSampler(0, "00000000:1B:00.0")
    c.start()
    t0 = time.time()
    time.sleep(0.03)
    t1 = time.time()
    c.stop()
    s = c.summary(t0, t1)
    assert s["source"] == "nvml 1 ms"
    assert s["samples"] >= 3
    assert 1700 <= s["sm_mhz"] <= 1720 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"]


def test_rejectable_reasons_are_named(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1200], 0x8 | 0x20 | 0x40))
    c = bench.ClockSampler(0)
    c.start()
    t0 = time.time()
    time.sleep(0.01)
    t1 = time.time()
    c.stop()
    assert c.summary(t0, t1)["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_sample_in_window_is_unsampled(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965], 0))
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.01)
    c.stop()
    later = time.time() + 10.0
    s = c.summary(later, later + 1.0)
    assert s["samples"] == 0 and s["reasons"] == ["unsampled"] and s["sm_mhz"] is None
