"""Deformable attention forward on NVFP4 values (and its full-precision twin) against the oracle.

Tolerance: the GPU forms the sampling coordinate x = fl(fl(loc * W) - 0.5) in FP32 (the oracle in
float64), an absolute error of at most 2u(W + 1) (u = 2^-24) that moves each bilinear weight by as
much, and it accumulates at most 4 corners x L x P products in FP32.  Per output channel:
    |out - oracle| <= (8 (W_max + H_max + 2) + 64) u * vmax * sum_{l,p} |w|
with vmax the largest value magnitude; a wrong code, scale, corner or level offset moves outputs by a
sizeable fraction of vmax * sum|w| and fails it."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu
U = 2.0 ** -24
SHAPES = [(6, 10), (3, 5), (2, 3), (1, 1)]


def _inputs(bs, heads, ch, nq, P, seed, dtype=torch.float32, shapes=SHAPES):
    g = torch.Generator().manual_seed(seed)
    nkeys = sum(h * w for h, w in shapes)
    value = (torch.randn((bs, nkeys, heads, ch), generator=g) * 2).to(dtype)
    loc = torch.rand((bs, nq, heads, len(shapes), P, 2), generator=g) * 1.3 - 0.15
    w = torch.rand((bs, nq, heads, len(shapes), P), generator=g)
    return value, loc, w


def _tol(value_f32, w, shapes):
    hw = max(max(h, wd) for h, wd in shapes)
    vmax = float(np.abs(value_f32).max())
    return (8 * (2 * hw + 2) + 64) * U * vmax * np.abs(w.numpy()).sum(axis=(-1, -2))[..., None]


def _host16(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("ch", [16, 32, 64])
def test_msda_nvfp4_matches_oracle(ch):
    bs, heads, nq, P = 2, 3, 9, 3
    value, loc, w = _inputs(bs, heads, ch, nq, P, seed=ch)
    codes, scales, g, _, _ = nv.quantize_ex(value.cuda().reshape(-1), want_f=False, want_sse=False)
    nkeys = value.shape[1]
    out = nv.msda_forward((codes.reshape(bs, nkeys, heads, ch // 2), scales.reshape(bs, nkeys, heads, ch // 16), g),
                          SHAPES, loc.cuda(), w.cuda())
    torch.cuda.synchronize()
    rc, rs, rg, _, _ = O.quantize(value.numpy().reshape(-1))
    vq = O.dequantize(rc, rs, rg).reshape(value.shape)
    ref = O.msda_forward(vq, SHAPES, loc.numpy(), w.numpy())
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert (err <= _tol(vq, w, SHAPES)).all(), float(err.max())
    # a wrong level offset or corner would be O(vmax * sum|w|): make sure the data exercises it
    assert np.abs(ref).max() > 0.1


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_msda_full_precision_twin_matches_oracle(dtype):
    bs, heads, ch, nq, P = 2, 2, 32, 11, 4
    value, loc, w = _inputs(bs, heads, ch, nq, P, seed=5, dtype=dtype)
    out = nv.msda_forward(value.cuda(), SHAPES, loc.cuda(), w.cuda())
    torch.cuda.synchronize()
    vf = value.float().numpy()
    ref = O.msda_forward(vf, SHAPES, loc.numpy(), w.numpy())
    err = np.abs(out.cpu().numpy().astype(np.float64) - ref)
    assert (err <= _tol(vf, w, SHAPES)).all(), float(err.max())


def test_msda_errors():
    value, loc, w = _inputs(1, 1, 32, 2, 2, seed=1)
    v = value.cuda()
    with pytest.raises(nv.NVFP4Error) as e:
        nv.msda_forward(v, [(6, 10), (3, 5)], loc.cuda()[:, :, :, :2].contiguous(), w.cuda()[:, :, :, :2].contiguous())
    assert e.value.status == -2          # level sizes do not add up to the keys
    v24 = torch.zeros((1, value.shape[1], 1, 24), device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.msda_forward(v24, SHAPES, loc.cuda(), w.cuda())
    assert e.value.status == -2          # 24 channels per head
    out = torch.empty(1 * 2 * 1 * 32 + 1, device="cuda")[1:].reshape(1, 2, 1, 32)
    with pytest.raises(nv.NVFP4Error) as e:
        nv.msda_forward(v, SHAPES, loc.cuda(), w.cuda(), out=out)
    assert e.value.status == -3          # output not 32-byte aligned


def test_msda_full_size_bev_sampled():
    """The C5 value maps [6, 30825, 8, 32] (FP16) with ScaleSearch NVFP4 values, 10000 queries per camera;
    sampled queries checked against the oracle on the oracle's own quantization."""
    value = W.bev_f16("cuda")                      # [6, 30825, 8, 32]
    bs, nkeys, heads, ch = value.shape
    loc, w = W.msda_inputs("cuda")
    codes, scales, g, _, _ = nv.quantize_ex(value.reshape(-1), want_f=False, want_sse=False)
    out = nv.msda_forward((codes.reshape(bs, nkeys, heads, ch // 2), scales.reshape(bs, nkeys, heads, ch // 16), g),
                          W.LEVELS, loc, w)
    torch.cuda.synchronize()
    vh = _host16(value.cpu())
    rc, rs, rg, _, _ = O.quantize(vh.reshape(-1), dtype=O.F16)
    assert g.item() == rg
    vq = O.dequantize(rc, rs, rg).reshape(bs, nkeys, heads, ch)
    rng = np.random.default_rng(2)
    qs = np.sort(rng.choice(loc.shape[1], 64, replace=False))
    loc_s, w_s = loc[:, qs].cpu(), w[:, qs].cpu()
    ref = O.msda_forward(vq, W.LEVELS, loc_s.numpy(), w_s.numpy())
    got = out[:, qs].cpu().numpy().astype(np.float64)
    tol = _tol(vq, w_s, W.LEVELS)
    assert (np.abs(got - ref) <= tol).all(), float(np.abs(got - ref).max())
