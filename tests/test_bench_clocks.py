"""bench.py's clock sampler against a fake NVML on CPU: the median SM clock,
the throttle reasons decoded from the clock-event bits, the no-NVML path.
The fake exposes read calls only, so any attempt to change a clock or a
limit would fail here (the sampler only reads)."""

import importlib.util
import os
import sys
import time
import types

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fake_nvml(clocks, reasons, fail_init=False):
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    state = {"i": 0}

    def init():
        if fail_init:
            raise RuntimeError("NVML Shared Library Not Found")

    def clock(handle, kind):
        assert handle == "h" and kind == nv.NVML_CLOCK_SM
        return clocks[min(state["i"], len(clocks) - 1)]

    def event_reasons(handle):
        r = reasons[min(state["i"], len(reasons) - 1)]
        state["i"] += 1
        return r

    nv.nvmlInit = init
    nv.nvmlDeviceGetHandleByUUID = lambda uuid: "h"
    nv.nvmlDeviceGetMaxClockInfo = lambda handle, kind: 1965
    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = event_reasons
    return nv


def _run(monkeypatch, nv, seconds=0.03):
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    b = _bench()
    cs = b.ClockSampler("GPU-fake")
    cs.start()
    time.sleep(seconds)
    return cs.stop()


def test_power_cap_is_kept_and_named(monkeypatch):
    nv = _fake_nvml([1965, 1965, 1950, 1965], [0, 0x4, 0x4, 0])
    out = _run(monkeypatch, nv)
    assert out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz"] == pytest.approx(1965.0)
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] >= 4


def test_hardware_slowdown_is_reported(monkeypatch):
    nv = _fake_nvml([1965, 1200, 1200, 1200, 1200], [0, 0x8, 0x8 | 0x40, 0x8, 0x8])
    out = _run(monkeypatch, nv)
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert out["sm_mhz"] == pytest.approx(1200.0)


def test_no_nvml_reports_why(monkeypatch):
    out = _run(monkeypatch, _fake_nvml([0], [0], fail_init=True), seconds=0.0)
    assert out["sm_mhz"] is None and out["samples"] == 0
    assert out["reasons"] and out["reasons"][0].startswith("no NVML")
