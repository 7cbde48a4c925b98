"""Host logic of bench.py that decides whether a measurement stands, checked on CPU: the clock
record (median SM clock, maximum, throttle reasons) from nvidia-smi lines and from a fake NVML, and
the recorded ncu traffic, which must read null once the kernel's sources differ from the captured
ones."""
import json
import os
import threading
import time

import pytest

import bench


def smi_line(sm, mx, active, hw=False, hw_th=False, sw_th=False, cap=False):
    f = lambda b: "Active" if b else "Not Active"
    return f"0, {sm}, {mx}, 812.5, {active}, {f(hw)}, {f(hw_th)}, {f(sw_th)}, {f(cap)}"


def test_clock_summary_of_nvidia_smi_lines():
    s = bench.ClockSampler(0)
    s.lines = [smi_line(1965, 1965, "0x0"), smi_line(1950, 1965, "0x4", cap=True),
               smi_line(1965, 1965, "0x0"), "", "garbage line", smi_line("[N/A]", 1965, "0x0")]
    r = s.summary()
    assert r["samples"] == 3 and r["sm_mhz"] == 1965.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]


def test_clock_summary_names_every_rejecting_reason():
    s = bench.ClockSampler(0)
    s.lines = [smi_line(1200, 1965, "0x8", hw=True), smi_line(1300, 1965, "0x40", hw_th=True),
               smi_line(1400, 1965, "0x20", sw_th=True)]
    r = s.summary()
    assert r["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert r["sm_mhz"] == 1300.0


def test_clock_summary_without_samples():
    r = bench.ClockSampler(0).summary()
    assert r == {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}


class FakeNvml:
    """The read-only NVML queries the sampler makes, answering from a script of samples."""
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8
    nvmlClocksEventReasonSwThermalSlowdown = 0x20
    nvmlClocksEventReasonHwThermalSlowdown = 0x40
    NVML_CLOCK_SM = 1

    def __init__(self, samples):
        self.samples, self.i = samples, 0
        self.calls = []

    def nvmlDeviceGetMaxClockInfo(self, h, which):
        self.calls.append("max")
        return 1965

    def nvmlDeviceGetClockInfo(self, h, which):
        self.calls.append("clock")
        return self.samples[min(self.i, len(self.samples) - 1)][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.samples[min(self.i, len(self.samples) - 1)][1]

    def nvmlDeviceGetPowerUsage(self, h):
        self.i += 1
        return 950000  # mW


def test_clock_sampler_polls_a_fake_nvml_until_stopped():
    nv = FakeNvml([(1965, 0x0), (1965, 0x4), (1890, 0x4 | 0x8)])
    s = bench.ClockSampler(0)
    t = threading.Thread(target=s._poll_nvml, args=(nv, object()), daemon=True)
    t.start()
    t0 = time.perf_counter()
    while len(s.lines) < 6 and time.perf_counter() - t0 < 5.0:
        time.sleep(0.002)
    s.stop.set()
    t.join(timeout=2.0)
    assert not t.is_alive()
    r = s.summary()
    assert r["samples"] >= 6 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert set(nv.calls) == {"max", "clock"}  # queries only: nothing is set


def test_recorded_traffic_reads_null_once_the_sources_change(tmp_path, monkeypatch):
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        rec = json.load(f)
    key, e = next(iter(rec.items()))
    assert bench.recorded_traffic(key) == e["bytes_per_launch"]  # the committed capture is current
    monkeypatch.setattr(bench, "sources_sha", lambda names: "0" * 16)
    assert bench.recorded_traffic(key) is None
    assert bench.recorded_traffic("no such kernel") is None


def test_sources_sha_depends_on_every_listed_file():
    a = bench.sources_sha(["chain.cu"])
    b = bench.sources_sha(["chain.cu", "gemv_core.cuh"])
    assert len(a) == 16 and a != b
    with pytest.raises(FileNotFoundError):
        bench.sources_sha(["no_such_file.cu"])


def test_cpu_info_reports_usable_cores():
    model, n = bench.cpu_info()
    assert n >= 1 and (model is None or isinstance(model, str))


def test_fp4_roofline_carries_the_probe_or_nulls(monkeypatch):
    monkeypatch.setattr(bench, "fp4_peaks", lambda: (6500.0, "test", 9000.0))
    monkeypatch.setattr(bench, "fp4_mma_probe", lambda: {"tflops": 8000.0, "status": 0})
    r = bench.roofline_fp4("k", 2e12, 1000.0)  # 2 TFLOP in 1 ms
    assert r["achieved"] == pytest.approx(2000.0) and r["frac"] == pytest.approx(2000 / 6500)
    assert r["probe_peak"] == 8000.0 and r["frac_of_probe"] == pytest.approx(0.25)
    monkeypatch.setattr(bench, "fp4_mma_probe", lambda: {"tflops": 8000.0, "status": 1})  # a wait gave up
    r = bench.roofline_fp4("k", 2e12, 1000.0)
    assert r["probe_peak"] is None and r["frac_of_probe"] is None and r["frac"] == pytest.approx(2000 / 6500)

    def boom():
        raise RuntimeError("no device")
    monkeypatch.setattr(bench, "fp4_mma_probe", boom)
    r = bench.roofline_fp4("k", 2e12, 1000.0)
    assert r["probe_peak"] is None and "no device" in r["probe"]["error"]


def test_hbm_roofline_prints_the_measured_and_the_spec_peak(monkeypatch):
    monkeypatch.setattr(bench, "peaks", lambda: (6558.1, "measured"))
    r = bench.roofline_hbm("k", 6.5581e9, 1000.0, traffic=123)  # 6.5581 GB in 1 ms
    assert r["achieved"] == pytest.approx(6558.1) and r["frac"] == pytest.approx(1.0)
    assert r["spec_peak"] == 8000.0 and r["frac_of_spec"] == pytest.approx(6558.1 / 8000.0)
    assert r["traffic"] == 123 and r["bound"] == "hbm" and r["unit"] == "GB/s"
