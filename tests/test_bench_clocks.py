"""The bench's clock record: NVML read every millisecond inside the timed windows (plus
one sample at each edge), throttle-reason bits mapped to names; without NVML, the
nvidia-smi fallback, which yields no record where nvidia-smi cannot run."""
import os
import sys
import time
import types

import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))


def fake_nvml(reasons_bits, fail_init=False):
    m = types.ModuleType("pynvml")
    m.NVML_CLOCK_SM = 1
    m.nvmlClocksEventReasonSwPowerCap = 0x4
    m.nvmlClocksEventReasonHwSlowdown = 0x8
    m.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    m.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    m.calls = {"clock": 0, "shutdown": 0}

    def init():
        if fail_init:
            raise RuntimeError("no NVML here")
    m.nvmlInit = init
    m.nvmlShutdown = lambda: m.calls.__setitem__("shutdown", m.calls["shutdown"] + 1)
    m.nvmlDeviceGetHandleByUUID = lambda uuid: ("handle", uuid)
    m.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        m.calls["clock"] += 1
        return 1965 if m.calls["clock"] % 2 else 1950
    m.nvmlDeviceGetClockInfo = clock
    m.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons_bits
    return m


@pytest.fixture
def bench_mod():
    import bench
    return bench


def test_nvml_window_samples(monkeypatch, bench_mod):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(0x4 | 0x1))   # power cap + idle bit
    clk = bench_mod.ClockSampler("GPU-00000000-0000-0000-0000-000000000000")
    clk.begin()
    clk.window_start()
    time.sleep(0.05)
    clk.window_stop()
    clk.window_start()
    clk.window_stop()
    d = clk.end()
    assert d["samples"] >= 4                      # edges of both windows at least
    assert d["sm_max_mhz"] == 1965.0
    assert 1950.0 <= d["sm_mhz"] <= 1965.0
    assert d["reasons"] == ["sw_power_cap"]
    assert d["source"].startswith("NVML")


def test_nvml_throttle_names(monkeypatch, bench_mod):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(0x8 | 0x20 | 0x40))
    clk = bench_mod.ClockSampler("GPU-x")
    clk.window_start()
    clk.window_stop()
    assert clk.end()["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_fallback_without_nvml(monkeypatch, bench_mod):
    monkeypatch.setitem(sys.modules, "pynvml", fake_nvml(0, fail_init=True))
    monkeypatch.setenv("PATH", "/nonexistent")          # no nvidia-smi either
    clk = bench_mod.ClockSampler("GPU-x")
    clk.begin()
    clk.window_start()
    clk.window_stop()
    assert clk.end() is None
