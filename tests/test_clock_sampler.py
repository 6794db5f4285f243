"""bench.py's clock sampler against a fake nvidia-smi on PATH: samples taken while the timed
region runs are summarised as the median SM clock, the maximum clock and the throttle reasons
that were active."""

import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_smi(tmp_path, lines):
    script = tmp_path / "nvidia-smi"
    body = "\n".join(f"echo '{l}'" for l in lines)
    script.write_text("#!/bin/bash\n" + body + "\nsleep 30\n")
    script.chmod(script.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def test_summary_median_and_reasons(tmp_path, monkeypatch):
    lines = ["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
             "0, 1900, 1965, 900.5, 0x4, Not Active, Not Active, Not Active, Active",
             "0, 1930, 1965, 950.0, 0x4, Not Active, Not Active, Not Active, Active"]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ["PATH"])
    monkeypatch.delenv("MISA_BENCH_LOG_DIR", raising=False)
    with bench.ClockSampler("GPU-fake", 0) as clk:
        time.sleep(0.3)
    s = clk.summary()
    assert s["sm_mhz"] == 1930 and s["sm_max_mhz"] == 1965 and s["samples"] == 3
    assert s["reasons"] == ["sw_power_cap"]


def test_unsampled_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))   # no nvidia-smi anywhere
    with bench.ClockSampler("GPU-fake", 1) as clk:
        pass
    assert clk.summary()["reasons"] == ["unsampled"]


def test_log_dir_keeps_the_samples(tmp_path, monkeypatch):
    lines = ["0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active"]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ["PATH"])
    monkeypatch.setenv("MISA_BENCH_LOG_DIR", str(tmp_path / "logs"))
    with bench.ClockSampler("GPU-fake", 2) as clk:
        time.sleep(0.3)
    assert (tmp_path / "logs" / "clocks_rank2.csv").exists()
    assert clk.summary()["samples"] == 1
