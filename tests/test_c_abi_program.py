"""libnvfp4 from plain C: tests/c_abi/roundtrip.c calls the C ABI with CUDA-runtime buffers (no Python,
no torch in that process) and compares every output byte with the oracle's C functions.  On CPU the
program must compile and link; on a B200 it runs."""
import os
import subprocess

import pytest

import nvfp4_block_scaled_11_b200 as nv
from oracle import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path) -> str:
    lib_dir = os.path.dirname(nv.library_path())
    ref_dir = os.path.dirname(O.build())
    exe = str(tmp_path / "roundtrip")
    cmd = ["gcc", "-std=c99", "-O2", "-Wall", "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "oracle"),
           "-I", os.path.join(CUDA, "include"), os.path.join(HERE, "c_abi", "roundtrip.c"), "-o", exe,
           "-L", lib_dir, "-lnvfp4", "-L", ref_dir, "-lnvfp4_ref", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-lm", f"-Wl,-rpath,{lib_dir}:{ref_dir}:{os.path.join(CUDA, 'lib64')}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert os.access(_build(tmp_path), os.X_OK)


@pytest.mark.gpu
def test_c_program_round_trip(tmp_path):
    r = subprocess.run([_build(tmp_path)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
