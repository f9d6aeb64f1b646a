"""Whole-tensor parity at the full sizes of the five workloads, in the launch configurations the benchmark
times: every code byte, scale byte, chosen offset, block SSE and dequantized value of the GPU equals the
oracle's (0 mismatches), g is bit-equal, and the aggregate MSE statistics agree (relative 1e-6; with every
block SSE bit-equal they agree exactly).  The oracle runs over block ranges in spawned worker processes on
the host cores (tests/fullsize.py).  C4 (2^30 FP32 elements) is checked for the three windows of its sweep;
its oracle work is about 700 core-seconds, a minute or so on a 16-core host."""
import os

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W
from oracle import oracle as O

from . import fullsize as FS

pytestmark = [pytest.mark.gpu, pytest.mark.timeout(1800)]

DT_CODE = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


def _dump(t: torch.Tensor, path: str, chunk: int = 1 << 28) -> str:
    """Write a device tensor's bytes to a file (in chunks, to bound host memory)."""
    flat = t.contiguous().view(-1).view(torch.uint8)
    with open(path, "wb") as fh:
        for i in range(0, flat.numel(), chunk):
            fh.write(flat[i:i + chunk].cpu().numpy().tobytes())
    return path


def _assert_clean(tot: dict, nb: int, keys=("codes", "scales", "f", "sse", "deq")):
    assert tot["blocks"] == nb
    for k in keys:
        if k in tot:
            assert tot[k] == 0, (k, tot[k], tot.get(k + "_first"))


def _linear_case(name, tmp_path, windows):
    torch.cuda.empty_cache()
    w = W.make(name, "cuda")
    x = w.x.reshape(-1).contiguous()
    n, dt = x.numel(), DT_CODE[x.dtype]
    nb = n // 16
    xpath = _dump(x, str(tmp_path / "x.bin"))
    rg = O.global_scale(O.tensor_amax(np.memmap(xpath, FS.NP_DTYPE[dt], "r", shape=(n,)), dt))
    res = {}
    for (f_lo, f_hi) in windows:
        # the two-pass quantize (its own amax pass), then f* and SSE with that g
        codes, scales, g = nv.quantize(x, f_lo, f_hi)
        assert g.item() == rg or (np.isnan(rg) and np.isnan(g.item()))
        _, _, _, bf, bs = nv.quantize_ex(x, f_lo, f_hi, gscale_in=g)
        paths = {"codes": _dump(codes, str(tmp_path / "c.bin")), "scales": _dump(scales, str(tmp_path / "s.bin")),
                 "f": _dump(bf, str(tmp_path / "f.bin")), "sse": _dump(bs, str(tmp_path / "e.bin"))}
        if (f_lo, f_hi) == (w.f_lo, w.f_hi):
            # the benchmark's step: the fused round trip, values in the input's dtype (and its codes)
            fo, fc, fs, fg = nv.quantize_dequantize(x, f_lo, f_hi, gscale_in=g)
            assert torch.equal(fc, codes) and torch.equal(fs, scales)
            paths["deq"] = _dump(fo, str(tmp_path / "d.bin"))
            del fo, fc, fs
        del codes, scales, bf, bs
        torch.cuda.synchronize()
        tot = FS.oracle_compare(xpath, dt, n, rg, f_lo, f_hi, paths, deq_dtype=dt)
        _assert_clean(tot, nb)
        res[(f_lo, f_hi)] = tot
    if x.dtype == torch.float32:
        # the FP32 dequantize of the default window's codes (the two-pass schedule) is bit-exact too
        codes, scales, g = nv.quantize(x, w.f_lo, w.f_hi)
        out = nv.dequantize(codes, scales, g, torch.float32)
        tot = FS.oracle_compare(xpath, dt, n, rg, w.f_lo, w.f_hi,
                                {"codes": _dump(codes, str(tmp_path / "c.bin")),
                                 "scales": _dump(scales, str(tmp_path / "s.bin")),
                                 "deq": _dump(out, str(tmp_path / "d.bin"))}, deq_dtype=0)
        _assert_clean(tot, nb)
    return res


@pytest.mark.parametrize("name", ["act_f32", "bev_f16"])
def test_whole_tensor_linear(name, tmp_path):
    _linear_case(name, tmp_path, [(-2, 6)])


def test_whole_tensor_act_bf16_histogram_and_mse(tmp_path):
    """C2: ScaleSearch [-2,6] against max-scaling {0}: every block's offset and SSE bit-equal to the
    oracle's, hence the per-offset histogram and the aggregate MSE reduction (here compared at 1e-6)."""
    res = _linear_case("act_bf16", tmp_path, [(-2, 6), (0, 0)])
    s, s0 = res[(-2, 6)]["sse_sum"], res[(0, 0)]["sse_sum"]
    w = W.make("act_bf16", "cuda")
    x = w.x.reshape(-1)
    g = nv.global_scale(nv.tensor_amax(x))
    _, _, _, bf, bs = nv.quantize_ex(x, -2, 6, gscale_in=g)
    _, _, _, _, bs0 = nv.quantize_ex(x, 0, 0, gscale_in=g)
    gpu_hist = torch.bincount(bf.to(torch.int64) + 128, minlength=256).cpu().numpy()
    assert np.array_equal(gpu_hist, res[(-2, 6)]["hist"])
    red_gpu = 1.0 - bs.double().sum().item() / bs0.double().sum().item()
    red_ref = 1.0 - s / s0
    assert red_ref > 0 and abs(red_gpu - red_ref) <= 1e-6 * abs(red_ref)


def test_whole_tensor_stream_f32_window_sweep(tmp_path):
    """C4: 2^30 FP32 elements, windows {0}, [-2,6] (with the fused round trip) and [-8,8]."""
    _linear_case("stream_f32", tmp_path, [(0, 0), (-2, 6), (-8, 8)])


def test_whole_tensor_kv_bf16(tmp_path):
    """C3: the whole KV layout of nvfp4_kv_mixed_dequantize (the benchmark's call) against the oracle's
    one-shot ref_kv_mixed: sink and recent tokens verbatim, g, every code and scale byte, and every
    dequantized (rotated, BF16) middle value."""
    torch.cuda.empty_cache()
    k = W.make("kv_bf16", "cuda").x
    B, H, T, D = k.shape
    deq = torch.empty(B * H * (T - 32) * D, dtype=torch.bfloat16, device="cuda")
    so, ro, codes, scales, g, _ = nv.kv_mixed_dequantize(k, 16, 16, True, -2, 6, mid_out=deq)
    torch.cuda.synchronize()
    kh = k.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    rso, rro, rc, rs, rg = O.kv_mixed(kh, 16, 16, 1, -2, 6)
    assert g.item() == rg
    assert np.array_equal(so.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1), rso.reshape(-1))
    assert np.array_equal(ro.cpu().contiguous().view(torch.int16).numpy().view(np.uint16).reshape(-1), rro.reshape(-1))
    gc, gs = codes.cpu().numpy().reshape(-1), scales.cpu().numpy().reshape(-1)
    assert int((gc != rc.reshape(-1)).sum()) == 0 and int((gs != rs.reshape(-1)).sum()) == 0
    rd = O.dequantize(rc.reshape(-1), rs.reshape(-1), rg, out_dtype=O.BF16)
    assert np.array_equal(deq.cpu().view(torch.int16).numpy().view(np.uint16), rd.view(np.uint16))
