"""Error paths that need a GPU process of their own (both switches are read once per process):
checked mode reports non-finite input as NVFP4_ERR_NONFINITE, and a CUDA launch error, injected on the
host by an invalid launch configuration, comes back as NVFP4_ERR_CUDA with the context still usable.
Neither faults the GPU: the poison is in-band and the bad launch is refused before it is enqueued."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(code: str, **env) -> str:
    r = subprocess.run([sys.executable, "-c", code], env={**os.environ, **env}, cwd=ROOT, capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    return r.stdout


def test_checked_mode_reports_nonfinite():
    out = _run("""
import torch, nvfp4_block_scaled_11_b200 as nv
x = torch.randn(4096, device="cuda")
codes, scales, g = nv.quantize(x)
print("finite ok", bool((scales != 0x7F).all()))
x[100] = float("nan")
try:
    nv.quantize(x)
    print("no error")
except nv.NVFP4Error as e:
    print("status", e.status)
k = torch.randn(1, 2, 64, 32, device="cuda").to(torch.bfloat16)
nv.kv_mixed(k)                                   # finite: no error
k[0, 1, 30, 3] = float("inf")                    # a middle token
try:
    nv.kv_mixed(k)
    print("kv no error")
except nv.NVFP4Error as e:
    print("kv status", e.status)
try:
    nv.quantize_dequantize(x)
    print("fused no error")
except nv.NVFP4Error as e:
    print("fused status", e.status)
""", NVFP4_CHECKED="1")
    assert "finite ok True" in out and "status -5" in out, out
    assert "kv status -5" in out and "fused status -5" in out, out


def test_injected_launch_error_is_reported_and_recoverable():
    out = _run("""
import torch, nvfp4_block_scaled_11_b200 as nv
x = torch.randn(4096, device="cuda")
codes, scales, g = nv.quantize(x)
try:
    nv.dequantize(codes, scales, g)
    print("no error")
except nv.NVFP4Error as e:
    print("status", e.status)
c2, s2, g2 = nv.quantize(x)          # other entry points still run on the same context
torch.cuda.synchronize()
print("after", torch.equal(c2, codes) and torch.equal(s2, scales))
""", NVFP4_FAULT_INJECT="launch")
    assert "status -4" in out and "after True" in out, out
