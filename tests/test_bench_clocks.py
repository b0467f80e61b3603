"""bench.py's clock record, checked on the CPU against a fake NVML: the
sampler polls the SM clock and the clock-event reasons, reports the median
under load and every reason seen, and only reads."""
import importlib
import sys
import time
import types


def _fake_nvml(clocks, reasons):
    nv = types.ModuleType("pynvml")

    class NVMLError(Exception):
        pass

    state = {"i": 0, "calls": []}
    nv.NVMLError = NVMLError
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    nv.nvmlInit = lambda: state["calls"].append("init")
    nv.nvmlShutdown = lambda: state["calls"].append("shutdown")

    def by_bus(bus):
        raise NVMLError("no such bus")
    nv.nvmlDeviceGetHandleByPciBusId = by_bus
    nv.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        state["i"] += 1
        return clocks[min(state["i"] - 1, len(clocks) - 1)]
    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetCurrentClocksEventReasons = \
        lambda h: reasons[min(state["i"] - 1, len(reasons) - 1)]
    return nv, state


def test_nvml_sampler_median_and_reasons(monkeypatch):
    clocks = [1965, 1950, 1400, 1410, 1420, 1430, 1440]
    reasons = [0, 0, 0x4, 0x4, 0x4, 0x4, 0x4]
    nv, state = _fake_nvml(clocks, reasons)
    monkeypatch.setitem(sys.modules, "pynvml", nv)
    bench = importlib.import_module("bench")
    s = bench.clock_sampler(0)
    assert isinstance(s, bench.NvmlClockSampler)
    s.start()
    time.sleep(0.05)
    out = s.stop()
    assert out["samples"] >= len(clocks)
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert 1400 <= out["sm_mhz"] <= 1440          # the median of a run that stays capped
    # only reads: init, polling, shutdown
    assert state["calls"] == ["init", "shutdown"]


def test_sampler_falls_back_without_nvml(monkeypatch):
    broken = types.ModuleType("pynvml")

    def fail():
        raise RuntimeError("no NVML here")
    broken.nvmlInit = fail
    monkeypatch.setitem(sys.modules, "pynvml", broken)
    bench = importlib.import_module("bench")
    assert isinstance(bench.clock_sampler(0), bench.ClockSampler)
