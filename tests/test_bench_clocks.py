"""Host-side check of the bench's clock sampler against a fake nvidia-smi that
prints one CSV sample per polling period (no GPU, no NVML)."""
import os
import stat
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

FAKE = r"""#!/usr/bin/env python3
import sys, time
period = 0.02
for i, a in enumerate(sys.argv):
    if a == "-lms":
        period = int(sys.argv[i + 1]) / 1000.0
t0 = time.time()
i = 0
while True:
    # a power-cap episode between 0.10 s and 0.20 s, full clocks otherwise
    t = time.time() - t0
    capped = 0.10 <= t < 0.20
    sm = 1800 if capped else 1965
    cap = "Active" if capped else "Not Active"
    print(f"{sm}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, {cap}", flush=True)
    i += 1
    time.sleep(period)
"""


@pytest.fixture
def fake_smi(tmp_path, monkeypatch):
    p = tmp_path / "nvidia-smi"
    p.write_text(FAKE)
    p.chmod(p.stat().st_mode | stat.S_IEXEC)
    monkeypatch.setenv("PATH", f"{tmp_path}{os.pathsep}{os.environ['PATH']}")
    return p


def test_samples_inside_the_region(fake_smi):
    import bench

    with bench.ClockSampler(0) as clk:
        assert clk.samples, "entering waits for the first sample"
        time.sleep(0.3)            # past the fake's capped episode
        clk.mark("start")
        time.sleep(0.15)
        clk.mark("end")
    s = clk.summary()
    assert s["basis"] == "inside the timed region"
    assert s["samples"] >= 4
    assert s["sm_mhz"] == 1965 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == []


def test_region_reasons_are_kept(fake_smi):
    import bench

    with bench.ClockSampler(0) as clk:
        t_first = clk.samples[0][0]
        # the fake caps from 0.10 s to 0.20 s after its start; put the region there
        while time.perf_counter() < t_first + 0.11:
            time.sleep(0.002)
        clk.mark("start")
        time.sleep(0.06)
        clk.mark("end")
    s = clk.summary()
    assert "sw_power_cap" in s["reasons"]
    assert s["sm_mhz"] == 1800


def test_short_region_takes_nearest_two(fake_smi):
    import bench

    with bench.ClockSampler(0) as clk:
        time.sleep(0.3)
        clk.mark("start")
        clk.mark("end")
    s = clk.summary()
    assert s["samples"] == 2
    assert s["basis"].startswith("the two samples nearest")


def test_no_nvidia_smi(tmp_path, monkeypatch):
    import bench

    monkeypatch.setenv("PATH", str(tmp_path))
    with bench.ClockSampler(0) as clk:
        clk.mark("start")
        clk.mark("end")
    assert clk.summary()["samples"] == 0
