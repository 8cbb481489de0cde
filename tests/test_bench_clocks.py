"""The benchmark's clock record and peak selection, on the host: the NVML
sampler runs against a stand-in NVML module (nothing touches a GPU), and the
peaks fall back to the pool's earlier figures without MEASURED_PEAKS.json."""
import importlib.util
import json
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _fake_nvml(clocks, reasons):
    """A stand-in for pynvml that replays a clock and reason sequence."""
    nv = types.ModuleType("pynvml")
    nv.NVML_CLOCK_SM = 1
    state = {"i": 0}

    class NVMLError(Exception):
        pass

    nv.NVMLError = NVMLError
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByPciBusId = lambda bus: ("pci", bus)
    nv.nvmlDeviceGetHandleByIndex = lambda i: ("idx", i)
    nv.nvmlDeviceGetMaxClockInfo = lambda h, kind: 1965

    def clock(h, kind):
        v = clocks[min(state["i"], len(clocks) - 1)]
        state["i"] += 1
        return v

    nv.nvmlDeviceGetClockInfo = clock
    nv.nvmlDeviceGetPowerUsage = lambda h: 612000  # milliwatts
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reasons
    return nv


def test_clock_sampler_reports_median_and_reasons(monkeypatch):
    bench = _bench()
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965, 1965, 990, 980, 975] + [975] * 200, 0x4))
    s = bench.ClockSampler(0, "00000000:1b:00.0")
    s.start()
    time.sleep(0.05)
    out = s.stop()
    assert out["source"].startswith("nvml")
    assert out["samples"] >= 3
    assert out["sm_max_mhz"] == 1965
    assert out["reasons"] == ["sw_power_cap"]
    assert 975 <= out["sm_mhz"] <= 1965
    assert out["power_w_max"] == 612.0


def test_clock_sampler_flags_slowdowns(monkeypatch):
    bench = _bench()
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml([1965], 0x8 | 0x40))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.02)
    out = s.stop()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert out["sm_mhz"] == 1965


def test_peaks_fallback_and_measured(tmp_path, monkeypatch):
    bench = _bench()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.measured_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0 and p["bf16_tflops"] == 1590.0
    (tmp_path / "MEASURED_PEAKS.json").write_text(json.dumps(
        {"hbm_gbs": 6532.5, "bf16_tflops": 1625.3, "bf16_tflops_sustained": 1400.0}))
    p = bench.measured_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6532.5 and p["bf16_tflops_sustained"] == 1400.0
