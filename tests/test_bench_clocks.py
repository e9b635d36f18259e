"""bench.py's clock sampler on the CPU, against a stand-in nvidia-smi that
prints one CSV sample every few milliseconds: only the samples inside the
marked region count, and the throttle reasons are collected from them."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fake_smi(tmp_path, lines):
    body = "\n".join(f'echo "{ln}"; sleep 0.01' for ln in lines)
    p = tmp_path / "nvidia-smi"
    p.write_text("#!/bin/sh\n" + body + "\nsleep 5\n")
    p.chmod(p.stat().st_mode | stat.S_IXUSR)
    return str(tmp_path)


def test_sampler_keeps_region_samples(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    idle = "345, 1965, 100.0, Not Active, Not Active, Not Active, Not Active"
    busy = "1800, 1965, 900.0, Not Active, Not Active, Not Active, Active"
    d = _fake_smi(tmp_path, [idle] * 3 + [busy] * 200)
    monkeypatch.setenv("PATH", d + os.pathsep + os.environ["PATH"])
    clk = bench.ClockSampler("GPU-fake").__enter__()   # waits 0.3 s: the idle lines arrive
    clk.mark_start()
    time.sleep(0.3)
    clk.mark_end()
    clk.__exit__(None, None, None)
    out = clk.summary()
    assert out["window"] == "timed regions"
    assert out["samples"] >= 5
    assert out["sm_mhz"] == 1800.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]


def test_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("PATH", str(tmp_path))       # no nvidia-smi anywhere
    clk = bench.ClockSampler("GPU-fake").__enter__()
    clk.mark_start()
    clk.mark_end()
    clk.__exit__(None, None, None)
    out = clk.summary()
    assert out["samples"] == 0 and out["sm_mhz"] is None and "error" in out
