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


def test_peak_follows_the_clocks():
    """Burst bf16 peak when the timed region ran at the maximum SM clock, the
    sustained (power-capped) figure otherwise."""
    bench = importlib.import_module("bench")
    pk = {"bf16": 1694.7, "bf16_sustained": 1438.2, "source": "measured"}
    peak, src = bench.bf16_peak_for_clocks(pk, {"sm_mhz": 1965, "sm_max_mhz": 1965})
    assert peak == 1694.7 and "burst" in src
    peak, src = bench.bf16_peak_for_clocks(pk, {"sm_mhz": 1514, "sm_max_mhz": 1965})
    assert peak == 1438.2 and "sustained" in src
    peak, _ = bench.bf16_peak_for_clocks(pk, {"sm_mhz": None, "sm_max_mhz": None})
    assert peak == 1438.2


def test_cpu_baseline_scales_setup_and_units_apart(monkeypatch):
    """The oracle sample converts only the sampled heads, times the per-head
    set-up apart from the per-block work, and scales each by its own count."""
    import numpy as np
    import torch
    bench = importlib.import_module("bench")

    class P:
        pass
    prob = P()
    g = torch.Generator().manual_seed(0)
    prob.batch, prob.hq, prob.hkv, prob.L, prob.d, prob.B, prob.S = 1, 4, 2, 256, 8, 32, 4
    prob.NB, prob.causal = 8, True
    prob.Q = torch.randn(1, 4, 256, 8, generator=g)
    prob.K = torch.randn(1, 2, 256, 8, generator=g)
    prob.V = torch.randn(1, 2, 256, 8, generator=g)
    prob.tau = np.full(4, 0.9, np.float32)
    cb = bench.oracle_sample(prob, [0, 3], n_blocks=4)
    assert cb["kind"] == "oracle" and cb["unit"] == "ms/layer" and cb["extrapolated"]
    assert cb["value"] > 0 and cb["measured_s"] > 0
    assert "query heads [0, 3] of 4 x 4 of 8 query blocks" in cb["sample"]


def test_launch_count_follows_the_dispatch():
    """gpu_launches per headline step: the scoring GEMM, then for r = B/S in
    1..32 the staged reduce, the selection filter and its fallback (the
    product path and the three calls alike), for other r the one-kernel fused
    reduce + select (product path) or the two-pass reduce and both selection
    kernels (three calls); then the schedule and the attention."""
    import bench
    assert bench.launches_per_step(8, False) == 6    # c2: S = 16, r = 8
    assert bench.launches_per_step(32, False) == 6   # S = 4
    assert bench.launches_per_step(4, True) == 6
    assert bench.launches_per_step(2, False) == 6    # S = 64
    assert bench.launches_per_step(64, False) == 4   # S = 2: fused wide kernel
    assert bench.launches_per_step(128, True) == 6
