"""The bench's clock sampler: samples are kept only when their timestamps fall inside the timed
region, and a region shorter than the sampling interval falls back to the nearest samples.
A stand-in nvidia-smi on PATH writes rows in the real query's format (no GPU needed)."""
import os
import stat
import sys
import time

import pytest

import bench

FAKE = r'''#!{py}
import datetime, sys, time
# rows of: timestamp, index, clocks.sm, clocks.max.sm, power.draw, reasons.active,
#          hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown, sw_power_cap
period = float({period})
while True:
    now = datetime.datetime.now().strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    sys.stdout.write(f"{{now}}, 0, 1965, 1965, 700.5, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    sys.stdout.flush()
    time.sleep(period)
'''


def _install(tmp_path, monkeypatch, period):
    p = tmp_path / "nvidia-smi"
    p.write_text(FAKE.format(py=sys.executable, period=period))
    p.chmod(p.stat().st_mode | stat.S_IXUSR)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")


def test_samples_inside_the_timed_region(tmp_path, monkeypatch):
    _install(tmp_path, monkeypatch, 0.01)
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.1)           # samples before the region are dropped
    s.begin()
    time.sleep(0.25)
    s.end()
    time.sleep(0.1)           # and after it
    c = s.stop()
    assert c["window"] == "timed region"
    assert c["sm_mhz"] == 1965.0 and c["sm_max_mhz"] == 1965.0 and c["reasons"] == []
    # about 25 rows at 10 ms; the 100 ms on either side would add about 20
    assert 5 <= c["samples"] <= 30


def test_region_shorter_than_the_interval_keeps_the_nearest(tmp_path, monkeypatch):
    _install(tmp_path, monkeypatch, 0.3)
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.05)
    s.begin()
    s.end()
    time.sleep(0.4)
    c = s.stop()
    assert c["window"] == "nearest"
    assert 1 <= c["samples"] <= 2 and c["sm_mhz"] == 1965.0


def test_missing_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    s = bench.ClockSampler(0)
    s.start()
    c = s.stop()
    assert c["sm_mhz"] is None and c["reasons"] == ["nvidia-smi unavailable"]
