"""Host-side checks of bench.py: the clock record (the NVML sampler driven by
a fake NVML module, no GPU) and the per-launch traffic records, which count
only while their kernel's sources are unchanged."""
import os
import sys
import time
import types

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_nvml(bits, mhz=1800, fail_uuid=False):
    def by_uuid(u):
        if fail_uuid:
            raise RuntimeError("unknown uuid")
        return "h"
    return types.SimpleNamespace(
        NVML_CLOCK_SM=1, NVMLError=RuntimeError, nvmlInit=lambda: None,
        nvmlDeviceGetHandleByUUID=by_uuid, nvmlDeviceGetHandleByIndex=lambda i: "h",
        nvmlDeviceGetMaxClockInfo=lambda h, c: 1965, nvmlDeviceGetClockInfo=lambda h, c: mhz,
        nvmlDeviceGetCurrentClocksEventReasons=lambda h: bits,
        nvmlClocksEventReasonHwSlowdown=0x8, nvmlClocksEventReasonHwThermalSlowdown=0x40,
        nvmlClocksEventReasonSwThermalSlowdown=0x20, nvmlClocksEventReasonSwPowerCap=0x4,
        nvmlClocksEventReasonHwPowerBrakeSlowdown=0x80)


def _sample(monkeypatch, fake):
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    sys.path.insert(0, ROOT)
    import bench
    s = bench.ClockSampler("GPU-0000", 0, period_s=0.001)
    s.start()
    time.sleep(0.03)
    return s.stop()


def test_power_cap_is_reported_and_clock_is_the_median(monkeypatch):
    rec = _sample(monkeypatch, _fake_nvml(0x4, mhz=1500))
    assert rec["sm_mhz"] == 1500 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"] and rec["samples"] >= 2


def test_thermal_and_hw_slowdown_bits(monkeypatch):
    rec = _sample(monkeypatch, _fake_nvml(0x8 | 0x40 | 0x20))
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_idle_bits_are_not_reasons(monkeypatch):
    rec = _sample(monkeypatch, _fake_nvml(0x1, fail_uuid=True))   # GPU-idle bit; handle found by index
    assert rec["reasons"] == []


def test_missing_nvml_is_reported(monkeypatch):
    broken = types.SimpleNamespace(nvmlInit=lambda: (_ for _ in ()).throw(OSError("no libnvidia-ml")))
    rec = _sample(monkeypatch, broken)
    assert "error" in rec and "libnvidia-ml" in rec["error"]


def test_traffic_record_scales_by_rows_and_goes_stale(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    rec = dict(bench.MEASURED_TRAFFIC["gate_score"])
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "probe", dict(rec, bytes=1000, rows=10))
    import hashlib
    h = hashlib.sha256()
    for f in rec["sources"]:
        h.update(open(os.path.join(ROOT, "learned_token_pruning_b200", "csrc", f), "rb").read())
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "probe", dict(rec, bytes=1000, rows=10, sha256=h.hexdigest()))
    assert bench.measured_traffic("probe", 40) == 4000
    monkeypatch.setitem(bench.MEASURED_TRAFFIC, "probe", dict(rec, bytes=1000, rows=10, sha256="0" * 64))
    assert bench.measured_traffic("probe", 40) is None
    assert bench.measured_traffic("no such kernel", 40) is None


def test_decode_extras_collects_each_workload_and_survives_a_failure():
    sys.path.insert(0, ROOT)
    import bench
    args = types.SimpleNamespace(steps=2, warmup=3)

    def fake_run(a, emit):
        assert a is args
        for name, rows, us in (("w_small", 2129, 14.8), ("w_large", 131137, 119.0)):
            emit({"mode": "decode", "workload": name, "cache_rows": rows, "us": us, "gbs": 1.0e3 / us,
                  "frac_hbm": 0.5, "ratio": 0.9, "l2": "flushed"})

    dec = bench.decode_extras(args, run=fake_run)
    assert set(dec) == {"w_small", "w_large"}
    assert dec["w_large"] == {"cache_rows": 131137, "us": 119.0, "gbs": 1.0e3 / 119.0, "frac_hbm": 0.5}

    def failing_run(a, emit):
        emit({"workload": "w_small", "cache_rows": 1, "us": 1.0, "gbs": 1.0, "frac_hbm": 0.1})
        raise RuntimeError("no device")

    assert bench.decode_extras(args, run=failing_run) == {"error": "RuntimeError: no device"}
