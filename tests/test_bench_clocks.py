"""bench.py's clock sampler on CPU, against a stand-in nvidia-smi that prints
fixed samples in the query format the sampler asks for."""
import os
import time

import bench

SAMPLES = """0, 1965, 1965, 910.5, 0x0000000000000004, Not Active, Not Active, Not Active, Active
0, 1950, 1965, 955.0, 0x0000000000000004, Not Active, Not Active, Not Active, Active
0, 345, 1965, 120.0, 0x0000000000000001, Not Active, Not Active, Not Active, Not Active
0, 1965, 1965, 930.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active
"""


def _fake_smi(tmp_path, text):
    exe = tmp_path / "nvidia-smi"
    exe.write_text("#!/bin/sh\ncat <<'EOF_SAMPLES'\n" + text + "EOF_SAMPLES\n")
    exe.chmod(0o755)
    return str(tmp_path)


def test_clock_summary_reads_reasons_and_loaded_median(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, SAMPLES) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as clk:
        time.sleep(0.5)
    s = clk.summary()
    assert s["reasons"] == ["sw_power_cap"]
    assert s["sm_max_mhz"] == 1965.0
    assert s["sm_mhz"] == 1965.0          # median of the loaded samples (the 345 MHz idle one left out)
    assert s["samples"] == 4


def test_clock_summary_flags_slowdowns(tmp_path, monkeypatch):
    text = "0, 1200, 1965, 700.0, 0x0000000000000048, Active, Not Active, Active, Not Active\n"
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, text) + os.pathsep + os.environ["PATH"])
    with bench.ClockSampler(0) as clk:
        time.sleep(0.3)
    assert clk.summary()["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))     # no nvidia-smi anywhere
    with bench.ClockSampler(0) as clk:
        pass
    assert clk.summary()["sm_mhz"] is None
