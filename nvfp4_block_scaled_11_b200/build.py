"""Build libnvfp4.so in-tree with nvcc for sm_100a.

    python -m nvfp4_block_scaled_11_b200.build [--force] [-v]

Two translation units, compiled to objects under _build/ and linked into one shared library with the
CUDA runtime linked statically:

* csrc/nvfp4_api.cu -- quantize / dequantize / Hadamard / KV kernels and the C ABI, compiled with
  -fmad=false so that no multiply-add is contracted where the definition rounds twice (fused
  operations are written out explicitly where they are wanted);
* csrc/gemm_nvfp4.cu -- the tensor-core NVFP4 product, built on the CUTLASS / CuTe headers (the
  include tree shipped with the flashinfer package, or NVFP4_CUTLASS_INCLUDE).

An object is rebuilt when one of its sources is newer than it.
"""
from __future__ import annotations

import importlib.util
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INC = os.path.join(ROOT, "include")
OBJ = os.path.join(PKG, "_build")
SO = os.path.join(PKG, "libnvfp4.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O2"]


def cutlass_include() -> list[str]:
    env = os.environ.get("NVFP4_CUTLASS_INCLUDE")
    roots = [env] if env else []
    for pkg, sub in (("flashinfer", ("data", "cutlass")), ("tilelang", ("3rdparty", "cutlass"))):
        spec = importlib.util.find_spec(pkg)
        if spec and spec.submodule_search_locations:
            roots.append(os.path.join(list(spec.submodule_search_locations)[0], *sub, "include"))
    for inc in roots:
        if inc and os.path.exists(os.path.join(inc, "cutlass", "detail", "sm100_blockscaled_layout.hpp")):
            util = os.path.join(os.path.dirname(inc), "tools", "util", "include")
            return ["-I", inc] + (["-I", util] if os.path.isdir(util) else [])
    raise RuntimeError("CUTLASS headers with sm100 block-scaled support not found (set NVFP4_CUTLASS_INCLUDE)")


def _units():
    hdr = os.path.join(INC, "nvfp4.h")
    cuh = [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith(".cuh")]
    api = os.path.join(CSRC, "nvfp4_api.cu")
    gemm = os.path.join(CSRC, "gemm_nvfp4.cu")
    return [
        (api, [api, hdr, *cuh], ["-fmad=false"]),
        (gemm, [gemm, hdr], ["--expt-relaxed-constexpr", "-diag-suppress", "20012", *cutlass_include()]),
    ]


def _stale(target: str, deps: list[str]) -> bool:
    return not os.path.exists(target) or os.path.getmtime(target) < max(os.path.getmtime(d) for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    os.makedirs(OBJ, exist_ok=True)
    objs = []
    for src, deps, extra in _units():
        obj = os.path.join(OBJ, os.path.basename(src)[:-3] + ".o")
        objs.append(obj)
        if force or _stale(obj, deps):
            cmd = [NVCC, *COMMON, *extra, "-I", INC, "-c", "-o", obj, src]
            if verbose:
                cmd.insert(1, "-Xptxas=-v")
                print(" ".join(cmd))
            subprocess.run(cmd, check=True)
    if force or _stale(SO, objs):
        cmd = [NVCC, *ARCH, "-shared", "-cudart", "static", "-o", SO, *objs]
        if verbose:
            print(" ".join(cmd))
        subprocess.run(cmd, check=True)
    return SO


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="-v" in sys.argv)
    print(SO)
