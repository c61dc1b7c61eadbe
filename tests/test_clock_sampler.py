"""bench.py's clock sampler against a fake nvidia-smi (CPU): samples are kept
when they arrive inside the marked timed region; a region shorter than the
sampling interval gets the nearest sample, labelled as such; throttle
reasons are read from the sampled columns."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

FAKE = r'''#!/usr/bin/env python3
import sys, time
# one CSV line every 10 ms: index, sm MHz (counts up from 1000), max MHz, power, reasons...
i = 0
while True:
    swp = "Active" if i % 2 else "Not Active"
    print(f"0, {1000 + i}, 1965, 500.0, 0x0, Not Active, Not Active, Not Active, {swp}", flush=True)
    i += 1
    time.sleep(0.01)
'''


def with_fake_smi(tmp_path, monkeypatch):
    exe = tmp_path / "nvidia-smi"
    exe.write_text(FAKE.replace("/usr/bin/env python3", sys.executable, 1))
    exe.chmod(exe.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ.get('PATH', '')}")


def test_samples_inside_the_marked_region(tmp_path, monkeypatch):
    with_fake_smi(tmp_path, monkeypatch)
    c = bench.ClockSampler(0)
    c.start()
    assert c.lines, "start() returns once a sample has arrived"
    time.sleep(0.1)
    c.mark_start()
    time.sleep(0.2)
    c.mark_end()
    time.sleep(0.1)
    r = c.stop()
    assert r["window"] == "timed region"
    assert 5 <= r["samples"] <= 40          # ~20 at 10 ms, none from the 0.1 s before or after
    assert r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap"]  # every other sample has it active
    first = float(c.lines[0][1].split(",")[1])
    assert r["sm_mhz"] >= first + 5          # the region's samples, not the first ones


def test_short_region_takes_the_nearest_sample(tmp_path, monkeypatch):
    with_fake_smi(tmp_path, monkeypatch)
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.05)
    c.t0 = c.t1 = time.time() - 1e-4  # a region far shorter than the interval, between two samples
    time.sleep(0.05)
    r = c.stop()
    assert r["samples"] == 1
    assert r["window"].startswith("nearest sample")


def test_no_sampler_means_no_clocks(monkeypatch):
    monkeypatch.setenv("PATH", "/nonexistent")
    c = bench.ClockSampler(0)
    c.start(wait_s=0.1)
    assert c.stop() is None
