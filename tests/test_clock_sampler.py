"""bench.py's clock sampler on CPU against a fake NVML: it polls while the timed region runs,
reports the median SM clock, the maximum clock and every throttle reason it saw, and only
reads (no call that sets a clock or any other setting exists on the fake)."""
import importlib.util
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fake_nvml(clocks, reasons):
    """A read-only NVML stand-in: successive samples cycle through `clocks` / `reasons`."""
    state = {"i": 0}

    def clock(h, which):
        assert h == "handle" and which == 0
        v = clocks[state["i"] % len(clocks)]
        return v

    def event_reasons(h):
        v = reasons[state["i"] % len(reasons)]
        state["i"] += 1
        return v

    return types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=lambda u: "handle" if u == "GPU-test" else None,
        nvmlDeviceGetHandleByIndex=lambda i: "handle",
        nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetMaxClockInfo=lambda h, which: 1965,
        nvmlDeviceGetCurrentClocksEventReasons=event_reasons,
        nvmlClocksEventReasonHwSlowdown=0x8,
        nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonSwThermalSlowdown=0x20,
        nvmlClocksEventReasonSwPowerCap=0x4)


def test_sampler_polls_nvml_during_a_short_region(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965, 1950, 1965], [0x0, 0x4, 0x1]))
    cs = _bench().ClockSampler("GPU-test")
    cs.start()
    time.sleep(0.05)  # a 50 ms timed region still yields many samples
    r = cs.stop()
    assert r["source"] == "nvml"
    assert r["samples"] >= 5
    assert r["sm_mhz"] == 1965 and r["sm_max_mhz"] == 1965
    assert r["reasons"] == ["sw_power_cap"]  # GpuIdle (0x1) is not a reason the bench reports


def test_sampler_reports_throttling(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1200], [0x8 | 0x40 | 0x20]))
    cs = _bench().ClockSampler("GPU-test")
    cs.start()
    time.sleep(0.02)
    r = cs.stop()
    assert r["sm_mhz"] == 1200
    assert r["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
