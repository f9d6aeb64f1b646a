"""Build libnvfp4.so in-tree with nvcc for sm_100a.

    python -m nvfp4_block_scaled_11_b200.build [--force]

The library is one CUDA translation unit (csrc/nvfp4_api.cu) compiled with -fmad=false so that no
multiply-add is ever contracted where the definition rounds twice; fused operations are written out
explicitly where they are wanted.  The CUDA runtime is linked statically.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
SO = os.path.join(PKG, "libnvfp4.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17", "-fmad=false",
    "-Xcompiler", "-fPIC,-O2", "-shared", "-cudart", "static",
]


def _sources():
    return [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".cu", ".cuh"))] + [
        os.path.join(ROOT, "include", "nvfp4.h")
    ]


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(SO):
        newest = max(os.path.getmtime(p) for p in _sources())
        if os.path.getmtime(SO) >= newest:
            return SO
    cmd = [NVCC, *FLAGS, "-I", os.path.join(ROOT, "include"), "-o", SO, os.path.join(CSRC, "nvfp4_api.cu")]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
        print(" ".join(cmd))
    subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(SO)
