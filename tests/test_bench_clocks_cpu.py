"""Host logic of bench.py's clock sampler, against a fake NVML (no GPU)."""
import time
import types

import bench


def _fake_nvml(clock_seq, reasons_seq):
    state = {"i": 0}

    def clock(h, which):
        i = min(state["i"], len(clock_seq) - 1)
        return clock_seq[i]

    def reasons(h):
        i = min(state["i"], len(reasons_seq) - 1)
        state["i"] += 1
        return reasons_seq[i]

    return types.SimpleNamespace(
        NVML_CLOCK_SM=0,
        nvmlDeviceGetClockInfo=clock,
        nvmlDeviceGetMaxClockInfo=lambda h, which: 1965,
        nvmlDeviceGetPowerUsage=lambda h: 900_000,
        nvmlDeviceGetCurrentClocksEventReasons=reasons,
    )


def test_samples_only_inside_timed_region_and_reason_bits(monkeypatch):
    fake = _fake_nvml([1965, 1800, 1700], [0x0, 0x4, 0x4 | 0x8])
    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", lambda self: (fake, object()))
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.02)
    s.begin()
    time.sleep(0.05)
    s.end()
    time.sleep(0.02)
    out = s.stop()
    assert out["source"].startswith("NVML")
    assert out["samples"] > 0
    assert out["sm_max_mhz"] == 1965.0
    # every sample counted lies inside [begin, end]
    assert all(s.t_begin <= t <= s.t_end for t, _, _, _ in s.samples if s._in_region(t))
    assert set(out["reasons"]) <= {"sw_power_cap", "hw_slowdown"}
    assert out["power_w_max"] == 900.0


def test_no_nvml_no_smi_reports_unavailable(monkeypatch):
    def boom(self):
        raise RuntimeError("no NVML")

    monkeypatch.setattr(bench.ClockSampler, "_nvml_handle", boom)
    monkeypatch.setattr(bench.subprocess, "Popen", lambda *a, **k: (_ for _ in ()).throw(OSError("no smi")))
    s = bench.ClockSampler(0)
    s.start()
    out = s.stop()
    assert out["sm_mhz"] is None and out["reasons"]
