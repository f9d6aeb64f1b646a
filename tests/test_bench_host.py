"""bench.py's host-side pieces on the CPU: the clock sampler's parsing of nvidia-smi's CSV (a stand-in
program on PATH prints the samples) and its fallback when the tool is missing."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_smi(tmp_path, lines):
    p = tmp_path / "nvidia-smi"
    body = "".join(f"echo '{ln}'\n" for ln in lines)
    p.write_text("#!/bin/sh\n" + body + "exec sleep 30\n")     # exec: terminate() ends the whole stand-in
    p.chmod(p.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def test_clock_sampler_parses_median_max_and_reasons(tmp_path, monkeypatch):
    lines = ["1965, 1965, 650.1, 0x0000000000000000", "1800, 1965, 990.0, 0x0000000000000004",
             "1900, 1965, 995.5, 0x0000000000000005", "[N/A], 1965, 1.0, 0x0"]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, lines) + os.pathsep + os.environ["PATH"])
    s = bench.ClockSampler(0)
    s.start()
    time.sleep(0.5)
    c = s.stop()
    assert c["samples"] == 3 and c["sm_mhz"] == 1900 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]                      # gpu_idle (bit 0) is not reported


def test_clock_sampler_without_the_tool(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))
    s = bench.ClockSampler(0)
    s.start()
    c = s.stop()
    assert c["samples"] == 0 and c["sm_mhz"] is None and c["reasons"]
