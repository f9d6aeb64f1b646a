"""Whole-tensor comparison of GPU outputs with the oracle at full size.

Blocks are independent given the tensor scale g, so the oracle's block quantizer runs over contiguous block
ranges in a pool of spawned worker processes on the host cores.  The input and the GPU's outputs are
memory-mapped files; each worker quantizes its range with the oracle, compares every code byte, scale byte,
chosen offset, block SSE and dequantized value with the GPU's, and reports mismatch counts, the first
mismatching block, the offset histogram and float64 sums of the block SSEs.  Test infrastructure only (no
torch import here: the workers load only numpy and the oracle)."""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np

NP_DTYPE = {0: np.float32, 1: np.uint16, 2: np.uint16}   # oracle dtype code -> element storage


def _first(mask: np.ndarray) -> int:
    i = np.flatnonzero(mask)
    return int(i[0]) if i.size else -1


def _range(job):
    (xpath, dt, n, b0, b1, g, f_lo, f_hi, paths, deq_dtype) = job
    from oracle import oracle as O
    x = np.memmap(xpath, dtype=NP_DTYPE[dt], mode="r", shape=(n,))
    rc, rs, rf, rse = O.quantize_blocks(x, b0, b1, g, f_lo, f_hi, dtype=dt)
    out = {"blocks": b1 - b0}
    gc = np.memmap(paths["codes"], np.uint8, "r")[8 * b0:8 * b1].reshape(-1, 8)
    bad = (gc != rc.reshape(-1, 8)).any(1)
    out["codes"], out["codes_first"] = int(bad.sum()), _first(bad) + b0 if bad.any() else -1
    gs = np.memmap(paths["scales"], np.uint8, "r")[b0:b1]
    bad = gs != rs
    out["scales"], out["scales_first"] = int(bad.sum()), _first(bad) + b0 if bad.any() else -1
    if paths.get("f") is not None:
        gf = np.memmap(paths["f"], np.int8, "r")[b0:b1]
        out["f"] = int((gf != rf).sum())
    if paths.get("sse") is not None:
        gse = np.memmap(paths["sse"], np.uint32, "r")[b0:b1]
        out["sse"] = int((gse != rse.view(np.uint32)).sum())
    out["hist"] = np.bincount(rf.astype(np.int64) + 128, minlength=256)
    out["sse_sum"] = float(rse.astype(np.float64).sum())
    if paths.get("deq") is not None:
        rd = O.dequantize(rc, rs, g, out_dtype=deq_dtype)
        width = np.uint32 if deq_dtype == 0 else np.uint16
        gd = np.memmap(paths["deq"], width, "r")[16 * b0:16 * b1]
        bad = gd != rd.view(width)
        out["deq"], out["deq_first"] = int(bad.sum()), _first(bad) // 16 + b0 if bad.any() else -1
    return out


def cores() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def oracle_compare(xpath: str, dt: int, n: int, g, f_lo: int, f_hi: int, paths: dict, deq_dtype: int = 0,
                   processes: int | None = None) -> dict:
    """Run the oracle over all n/16 blocks of the memory-mapped input and compare with the GPU outputs in
    `paths` (codes, scales and optionally f, sse, deq).  Returns summed mismatch counts, the smallest
    mismatching block per output, the offset histogram (index f + 128) and the float64 SSE sum."""
    nb = n // 16
    procs = processes or cores()
    nchunk = max(1, min(nb, 8 * procs))
    edges = [nb * i // nchunk for i in range(nchunk + 1)]
    jobs = [(xpath, dt, n, edges[i], edges[i + 1], float(g), f_lo, f_hi, paths, deq_dtype)
            for i in range(nchunk) if edges[i + 1] > edges[i]]
    with mp.get_context("spawn").Pool(procs) as pool:
        parts = pool.map(_range, jobs, chunksize=1)
    tot = {"blocks": 0, "hist": np.zeros(256, np.int64), "sse_sum": 0.0}
    for p in parts:
        for k, v in p.items():
            if k.endswith("_first"):
                if v >= 0:
                    tot[k] = v if tot.get(k, -1) < 0 else min(tot[k], v)
                else:
                    tot.setdefault(k, -1)
            else:
                tot[k] = tot.get(k, 0) + v
    return tot
