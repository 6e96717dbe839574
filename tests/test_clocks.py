"""The clock record every published number carries (streaming_causal_video_timestep_b200/clocks.py),
on the host: ClockSampler against a stand-in nvidia-smi that prints fixed samples, and the rule that
rejects hardware or thermal slowdowns but keeps the power cap.  Nothing here touches a GPU."""
import os
import stat
import sys
import time

from streaming_causal_video_timestep_b200.clocks import ClockSampler, clock_ok

# index, clocks.sm, clocks.max.sm, power.draw, active, hw_slowdown, hw_thermal, sw_thermal, sw_power_cap
SAMPLES = [
    "0, 1500, 1965, 990.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    "0, 1560, 1965, 998.7, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    "0, 1530, 1965, 1000.2, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
    "garbled line",
    "0, N/A, 1965, 1000.2, 0x0, Not Active, Not Active, Not Active, Not Active",
]


def _fake_smi(tmp_path, lines):
    script = tmp_path / "nvidia-smi"
    body = "\n".join(f"print({ln!r}, flush=True)" for ln in lines)
    script.write_text(f"#!{sys.executable}\nimport time\n{body}\ntime.sleep(30)\n")
    script.chmod(script.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def test_sampler_record_from_samples(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, SAMPLES) + os.pathsep + os.environ.get("PATH", ""))
    c = ClockSampler(0, interval_ms=100)
    c.start()
    deadline = time.time() + 10
    while len(c.lines) < len(SAMPLES) and time.time() < deadline:
        time.sleep(0.05)
    rec = c.stop()
    assert rec["samples"] == 3                       # the garbled and the N/A lines are skipped
    assert rec["sm_mhz"] == 1530.0                   # median of 1500, 1560, 1530
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["reasons"] == ["sw_power_cap"]
    assert clock_ok(rec)


def test_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))        # an empty directory: no nvidia-smi
    c = ClockSampler(0)
    c.start()
    rec = c.stop()
    assert rec["sm_mhz"] is None and rec["reasons"] == ["nvidia-smi unavailable"]


def test_slowdowns_reject_a_number_and_the_power_cap_does_not():
    assert clock_ok({"reasons": []})
    assert clock_ok({"reasons": ["sw_power_cap"]})
    for bad in ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"):
        assert not clock_ok({"reasons": ["sw_power_cap", bad]})
