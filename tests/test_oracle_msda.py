"""Pins for the oracle's multi-scale deformable attention forward.

The bilinear sampling at loc * size - 0.5 with zero padding is exactly torch's grid_sample (bilinear,
zeros, align_corners=False) at grid = 2 loc - 1, so per level the oracle must equal that library
routine weighted by the attention weights.  Plus closed forms: a pixel centre returns the pixel, a
location off the map contributes nothing, and the output is linear in the weights."""
import numpy as np
import torch
import torch.nn.functional as F

from oracle import oracle as O

SHAPES = [(6, 10), (3, 5), (2, 3)]


def _case(seed, bs=2, heads=3, ch=4, nq=7, P=3, lo=-0.1, hi=1.1):
    rng = np.random.default_rng(seed)
    nkeys = sum(h * w for h, w in SHAPES)
    value = rng.standard_normal((bs, nkeys, heads, ch)).astype(np.float32)
    loc = rng.uniform(lo, hi, (bs, nq, heads, len(SHAPES), P, 2)).astype(np.float32)
    w = rng.uniform(0, 1, (bs, nq, heads, len(SHAPES), P)).astype(np.float32)
    return value, loc, w


def _grid_sample_reference(value, loc, w):
    bs, nkeys, heads, ch = value.shape
    _, nq, _, L, P, _ = loc.shape
    v = torch.from_numpy(value).double()
    out = torch.zeros((bs, nq, heads, ch), dtype=torch.float64)
    start = 0
    for l, (H, W) in enumerate(SHAPES):
        vl = v[:, start:start + H * W].reshape(bs, H, W, heads, ch).permute(0, 3, 4, 1, 2).reshape(bs * heads, ch, H, W)
        g = torch.from_numpy(loc[:, :, :, l]).double().permute(0, 2, 1, 3, 4).reshape(bs * heads, nq, P, 2) * 2 - 1
        s = F.grid_sample(vl, g, mode="bilinear", padding_mode="zeros", align_corners=False)   # [bs*heads, ch, nq, P]
        wl = torch.from_numpy(w[:, :, :, l]).double().permute(0, 2, 1, 3).reshape(bs * heads, 1, nq, P)
        out += (s * wl).sum(-1).reshape(bs, heads, ch, nq).permute(0, 3, 1, 2)
        start += H * W
    return out.numpy()


def test_msda_oracle_matches_grid_sample():
    for seed in range(3):
        value, loc, w = _case(seed)
        got = O.msda_forward(value, SHAPES, loc, w)
        ref = _grid_sample_reference(value, loc, w)
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_msda_pixel_centre_and_outside():
    shapes = [(4, 8), (2, 4)]                       # power-of-two sizes: pixel centres are exact floats
    rng = np.random.default_rng(5)
    value = rng.standard_normal((1, 4 * 8 + 2 * 4, 1, 2)).astype(np.float32)
    loc = rng.uniform(0, 1, (1, 2, 1, 2, 2, 2)).astype(np.float32)
    w = np.zeros((1, 2, 1, 2, 2), np.float32)
    # query 0: level 1, point 0 at the centre of pixel (row 1, column 3) with weight 1
    loc[0, 0, 0, 1, 0] = [(3 + 0.5) / 4, (1 + 0.5) / 2]
    w[0, 0, 0, 1, 0] = 1.0
    # query 1: one point off the map (x * W - 0.5 < -1) with weight 1
    loc[0, 1, 0, 0, 0] = [-0.2, 0.5]
    w[0, 1, 0, 0, 0] = 1.0
    out = O.msda_forward(value, shapes, loc, w)
    key = 4 * 8 + 1 * 4 + 3
    assert np.array_equal(out[0, 0, 0], value[0, key, 0].astype(np.float64))
    assert not out[0, 1].any()


def test_msda_linear_in_weights():
    value, loc, w = _case(7)
    a = O.msda_forward(value, SHAPES, loc, w)
    b = O.msda_forward(value, SHAPES, loc, (2 * w).astype(np.float32))
    assert np.allclose(b, 2 * a, rtol=1e-12, atol=0)
