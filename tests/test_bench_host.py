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


def test_captured_traffic_scales_and_expires(tmp_path, monkeypatch):
    """The committed DRAM record is scaled to a launch by elements, and reads as None once any of the
    kernel's sources differs from what was hashed at capture time."""
    import hashlib
    import json
    (tmp_path / "profiles").mkdir()
    (tmp_path / "k.cuh").write_text("kernel source v1\n")
    h = hashlib.sha256(b"kernel source v1\n").hexdigest()
    rec = {"K": {"source_sha256": h, "source_files": ["k.cuh"], "captured_elements": 1000,
                 "dram_bytes_read": 3000, "dram_bytes_write": 1000}}
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("K", 5000) == 20000
    assert bench.captured_traffic("other", 5000) is None
    (tmp_path / "k.cuh").write_text("kernel source v2\n")
    assert bench.captured_traffic("K", 5000) is None
