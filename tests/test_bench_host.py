"""Host-side logic of bench.py that needs no GPU: the clock record (nvidia-smi samples kept only
inside the timed window, throttle reasons, median) and the traffic record's source check."""
from __future__ import annotations

import os
import stat
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _line(sm, mx=1965, power_cap="Not Active", thermal="Not Active"):
    return f"0, {sm}, {mx}, 900.00, 0x0000000000000004, Not Active, Not Active, {thermal}, {power_cap}"


def test_summary_keeps_only_the_timed_window():
    lines = [(10.0, _line(1200)),                      # idle, before the window
             (11.00, _line(1900, power_cap="Active")),
             (11.05, _line(1950)),
             (11.10, _line(1965)),
             (13.0, _line(800, thermal="Active"))]     # after the window
    rec = bench.ClockSampler.summarise(lines, 11.0, 11.1, 0.05)
    assert rec["samples"] == 3
    assert rec["sm_mhz"] == 1950 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]


def test_summary_of_a_window_shorter_than_the_interval_uses_the_nearest_sample():
    lines = [(10.0, _line(1500)), (10.5, _line(1940)), (12.0, _line(1700))]
    rec = bench.ClockSampler.summarise(lines, 10.52, 10.53, 0.005)
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1940


def test_summary_skips_malformed_lines():
    lines = [(1.0, "garbage"), (1.0, "0, [N/A], 1965, 1, 0, a, b, c, d"), (1.0, _line(1800))]
    rec = bench.ClockSampler.summarise(lines, None, None, 0.05)
    assert rec["samples"] == 1 and rec["sm_mhz"] == 1800 and rec["reasons"] == []


def test_sampler_reads_a_fake_nvidia_smi(tmp_path, monkeypatch):
    # a stand-in for nvidia-smi on PATH: prints one sample line every 10 ms until killed
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nwhile true; do\n  echo '" + _line(1965, power_cap="Active") +
                    "'\n  sleep 0.01\ndone\n")
    fake.chmod(fake.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ["PATH"])
    s = bench.ClockSampler(0, interval_ms=10)
    s.start()
    time.sleep(0.3)
    t0 = time.time()
    time.sleep(0.2)
    t1 = time.time()
    time.sleep(0.1)
    rec = s.stop(t0, t1)
    assert rec["samples"] >= 3
    assert rec["sm_mhz"] == 1965 and rec["reasons"] == ["sw_power_cap"]


def test_traffic_record_is_dropped_when_the_kernel_code_changes(monkeypatch):
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0000000000000000")
    assert bench.committed_traffic("full_61") is None
