"""Host logic of bench.py's clock sampler, with a stand-in for the NVML poller (no GPU)."""
import time

import bench

# prints what the NVML poller prints: a max line, then t,sm,power,reasons lines
FAKE_POLLER = r"""
import sys, time
print("max,1965", flush=True)
i = 0
while True:
    bits = [0x0, 0x4, 0x4 | 0x8][min(i, 2)]
    print("%.6f,%d,%.1f,%d" % (time.monotonic(), [1965, 1800, 1700][min(i, 2)], 900.0, bits), flush=True)
    i += 1
    time.sleep(0.001)
"""


def test_samples_only_inside_timed_region_and_reason_bits(monkeypatch):
    monkeypatch.setattr(bench, "SAMPLER_SRC", FAKE_POLLER)
    s = bench.ClockSampler(0)
    s.start()
    assert s.mode == "nvml" and s.max_mhz == 1965.0
    time.sleep(0.05)
    s.begin()
    time.sleep(0.1)
    s.end()
    time.sleep(0.05)
    out = s.stop()
    assert out["source"].startswith("NVML")
    assert out["samples"] > 0
    # only samples stamped inside [begin, end] are counted
    stamped = [float(ln.split(",")[0]) for _, ln in s.lines if ln.count(",") == 3]
    assert out["samples"] == sum(1 for t in stamped if s.t_begin <= t <= s.t_end) < len(stamped)
    assert out["sm_max_mhz"] == 1965.0
    assert set(out["reasons"]) <= {"sw_power_cap", "hw_slowdown"}
    assert out["power_w_max"] == 900.0


def test_no_poller_no_smi_reports_unavailable(monkeypatch):
    def no_exec(*a, **k):
        raise OSError("cannot start")

    monkeypatch.setattr(bench.subprocess, "Popen", no_exec)
    s = bench.ClockSampler(0)
    s.start()
    out = s.stop()
    assert out["sm_mhz"] is None and out["reasons"]
