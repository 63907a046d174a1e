"""Host-side pieces of bench.py, on CPU: the ncu traffic lookup and the clock sampler."""
import sys
import time
import types

import bench


def test_profiled_traffic_follows_the_kernel_source(tmp_path, monkeypatch):
    (tmp_path / "k.cu").write_text("__global__ void k() {}\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.source_sha(["k.cu"])
    (tmp_path / "profiles" / "k.md").write_text(f"source_sha: {sha}\ntraffic_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic(["k.cu"], "k.md") == 12345.0
    (tmp_path / "k.cu").write_text("__global__ void k() { }\n")      # the kernel changed since the capture
    assert bench.profiled_traffic(["k.cu"], "k.md") is None
    assert bench.profiled_traffic(["k.cu"], "missing.md") is None


def _fake_nvml(reason_bits):
    nv = types.SimpleNamespace()
    nv.NVML_CLOCK_SM = 1
    nv.nvmlClocksEventReasonHwSlowdown = 0x8
    nv.nvmlClocksEventReasonHwThermalSlowdown = 0x40
    nv.nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nv.nvmlClocksEventReasonSwPowerCap = 0x4
    clocks = iter([1800, 1965, 1965, 1900] + [1965] * 100000)
    nv.nvmlInit = lambda: None
    nv.nvmlDeviceGetHandleByUUID = lambda u: (_ for _ in ()).throw(RuntimeError("no uuid"))
    nv.nvmlDeviceGetHandleByIndex = lambda i: ("gpu", i)
    nv.nvmlDeviceGetMaxClockInfo = lambda h, c: 1965
    nv.nvmlDeviceGetClockInfo = lambda h, c: next(clocks)
    nv.nvmlDeviceGetCurrentClocksEventReasons = lambda h: reason_bits
    return nv


def test_clock_sampler_reports_median_and_named_reasons(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", _fake_nvml(0x4 | 0x8))
    cs = bench.ClockSampler(types.SimpleNamespace(index=0))
    time.sleep(0.05)
    out = cs.stop()
    assert out["sm_max_mhz"] == 1965 and out["samples"] >= 1
    assert out["sm_mhz"] in (1800, 1900, 1965)
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]


def test_clock_sampler_without_nvml_reports_nothing(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)   # import fails
    assert bench.ClockSampler(types.SimpleNamespace(index=0)).stop() is None
