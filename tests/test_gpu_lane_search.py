"""The three launch shapes of the ScaleSearch quantizers -- one offset per lane (a half warp or a warp
per block), a few offsets per lane (4 or 8 lanes per block) and a thread per block (the certified fast
score) -- each checked bit-exactly against the oracle on the same inputs, through every source mode
that reaches them (linear, KV with and without rotation, appended KV rows, transposed columns, fused
round trips).  The shape is forced with `search_policy` (bounds on the block count of each shape)."""
import contextlib

import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W
from oracle import oracle as O

pytestmark = pytest.mark.gpu

HUGE = 1 << 40
PATHS = {"lane1": (HUGE, HUGE), "lanes": (0, HUGE), "wide": (0, 0)}
SHAPES = list(PATHS)
DT = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}


@contextlib.contextmanager
def path(name):
    prev = nv.search_policy(*PATHS[name])
    try:
        yield
    finally:
        nv.search_policy(*prev)


def _host(t):
    t = t.cpu().contiguous()
    if t.dtype == torch.float32:
        return t.numpy()
    return t.view(torch.int16).numpy().view(np.uint16)


def same_f32(a, b):
    """Bit-equal FP32 arrays, NaN payloads aside (a poisoned block's SSE or values are NaN)."""
    a, b = np.asarray(a, np.float32).reshape(-1), np.asarray(b, np.float32).reshape(-1)
    nan = np.isnan(a)
    return np.array_equal(nan, np.isnan(b)) and np.array_equal(a[~nan].view(np.uint32), b[~nan].view(np.uint32))


def same_16(a, b, dtype):
    """Bit-equal BF16 / FP16 arrays (as uint16), NaN payloads aside."""
    a, b = np.asarray(a, np.uint16).reshape(-1), np.asarray(b, np.uint16).reshape(-1)
    to = torch.bfloat16 if dtype == torch.bfloat16 else torch.float16
    nan = torch.from_numpy(a.view(np.int16)).view(to).float().isnan().numpy()
    nb = torch.from_numpy(b.view(np.int16)).view(to).float().isnan().numpy()
    return np.array_equal(nan, nb) and np.array_equal(a[~nan], b[~nan])


def _special(g):
    """Blocks that reach every branch of the search under the tensor scale g: zero, NaN and Inf blocks
    (poisoned alone, g fixed), exactly representable blocks, single-element blocks (ties at SSE 0),
    blocks far above the tensor range (default code saturates, the window runs past code 126), blocks
    so small that the window falls below code 1, and subnormal magnitudes."""
    rng = np.random.default_rng(7)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float32)
    rows = [np.zeros(16, np.float32)]
    r = rng.standard_normal(16).astype(np.float32)
    r[5] = np.nan
    rows.append(r)
    r = rng.standard_normal(16).astype(np.float32)
    r[11] = -np.inf
    rows.append(r)
    for s in (g * 8.0, g * 64.0, g * 448.0):
        rows.append((rng.choice(grid, 16) * rng.choice([-1, 1], 16) * s).astype(np.float32))
    for v in (1.0, 3.0, 0.75, 1e-3):
        r = np.zeros(16, np.float32)
        r[rng.integers(16)] = v
        rows.append(r)
    for s in (1e3, 1e6, 1e-6, 1e-20, 1e-40):
        rows.append((rng.standard_normal(16) * s).astype(np.float32))
    return np.concatenate(rows)


def _check_quantize(x, f_lo, f_hi, gscale_in=None):
    gin = None if gscale_in is None else torch.tensor([gscale_in], dtype=torch.float32, device="cuda")
    c, s, g, bf, bs = nv.quantize_ex(x, f_lo, f_hi, gscale_in=gin)
    torch.cuda.synchronize()
    rc, rs, rg, rbf, rbs = O.quantize(_host(x).reshape(-1), f_lo, f_hi, dtype=DT[x.dtype], gscale_in=gscale_in)
    if g is not None:
        assert same_f32(g.cpu().numpy(), [rg])
    assert np.array_equal(s.cpu().numpy(), rs)
    assert np.array_equal(c.cpu().numpy(), rc)
    assert np.array_equal(bf.cpu().numpy(), rbf)
    assert same_f32(bs.cpu().numpy(), rbs)


@pytest.mark.parametrize("name", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("window", [(0, 0), (-2, 6), (-8, 8), (-3, 3), (-15, 16), (-20, 20)])
def test_linear_both_paths(name, dtype, window):
    x = W.stream_f32("cpu", scale=3000 * 16 / 2 ** 30)[: 3000 * 16 - 48].to(dtype)   # 2997 blocks
    with path(name):
        _check_quantize(x.cuda(), *window)
        sp = torch.from_numpy(_special(0.01)).to(dtype)
        _check_quantize(sp.cuda(), *window, gscale_in=0.01)


@pytest.mark.parametrize("name", SHAPES)
@pytest.mark.parametrize("nblocks", [1, 7, 15, 17, 33, 63, 65, 1003])
def test_ragged_group_counts(name, nblocks):
    """Launches whose block count leaves a CTA partly empty (a 256-thread CTA holds 16 blocks in
    half-warp groups, 8 in warp groups, 64 in groups of 4 lanes, 32 in groups of 8)."""
    g = torch.Generator().manual_seed(nblocks)
    x = torch.randn(nblocks * 16, generator=g) * 3.0
    with path(name):
        for window in ((-2, 6), (-8, 8)):
            _check_quantize(x.cuda(), *window)


@pytest.mark.parametrize("name", SHAPES)
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("window", [(0, 0), (-2, 6), (-8, 8)])
def test_fused_round_trip_both_paths(name, dtype, window):
    x = torch.cat([W.act_bf16("cpu", scale=4 / 8192, cols=1024).float().reshape(-1),
                   torch.from_numpy(_special(0.01))]).to(dtype)
    with path(name):
        for gin in (None, 0.01):
            gt = None if gin is None else torch.tensor([gin], dtype=torch.float32, device="cuda")
            out, c, s, g = nv.quantize_dequantize(x.cuda(), *window, gscale_in=gt)
            torch.cuda.synchronize()
            rc, rs, rg, _, _ = O.quantize(_host(x).reshape(-1), *window, dtype=DT[dtype], gscale_in=gin)
            assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
            rd = O.dequantize(rc, rs, rg, out_dtype=DT[dtype])
            got = _host(out).reshape(-1)
            if dtype == torch.float32:
                assert same_f32(got, rd)
            else:
                assert same_16(got, rd, dtype)


def _u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("name", SHAPES)
@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("window", [(-2, 6), (-8, 8), (0, 0)])
def test_kv_mixed_and_fused_both_paths(name, rotate, window):
    k = W.kv_bf16("cpu", scale=80 / 32768, heads=3, head_dim=64)          # [1, 3, 80, 64]
    so, ro, rc, rs, rg = O.kv_mixed(_u16(k), 16, 16, int(rotate), *window)
    with path(name):
        sk, rk, c, s, g = nv.kv_mixed(k.cuda(), 16, 16, rotate, *window)
        torch.cuda.synchronize()
        assert g.item() == rg
        assert np.array_equal(c.cpu().numpy(), rc) and np.array_equal(s.cpu().numpy(), rs)
        *_, c2, s2, g2, mid = nv.kv_mixed_dequantize(k.cuda(), 16, 16, rotate, *window)
        torch.cuda.synchronize()
        assert np.array_equal(c2.cpu().numpy(), rc) and np.array_equal(s2.cpu().numpy(), rs)
        rd = O.dequantize(rc.reshape(-1), rs.reshape(-1), rg, out_dtype=1)
        assert np.array_equal(_u16(mid).reshape(-1), rd.reshape(-1))


@pytest.mark.parametrize("name", SHAPES)
@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("tile", [False, True])
def test_kv_append_both_paths(name, rotate, tile):
    k = W.kv_decode_keys("cpu", n=40, heads=3, head_dim=128)              # [BH=3, 40, 128]
    BH, T, D = k.shape
    first, n, cap, t0 = 5, 16, 300, 120                                   # rows 120..135 cross a tile
    g = torch.tensor([0.0031], dtype=torch.float32)
    codes = torch.full((BH, cap, D // 2), 0xAA, dtype=torch.uint8, device="cuda")
    nsf = nv.sf_mma_bytes(cap, D, BH) if tile else BH * cap * (D // 16)
    scales = torch.full((nsf,), 0xAA, dtype=torch.uint8, device="cuda")
    with path(name):
        nv.kv_append(k.cuda(), first, n, g.cuda(), codes, scales, t0, rotate=rotate, tile_layout=tile)
        torch.cuda.synchronize()
    rc = np.full((BH, cap, D // 2), 0xAA, np.uint8)
    rs = np.full((BH, cap, D // 16), 0xAA, np.uint8)
    O.kv_append(_u16(k), first, n, g.item(), rc, rs, t0, rotate=int(rotate))
    assert np.array_equal(codes.cpu().numpy(), rc)
    if tile:
        want = np.full(nsf, 0xAA, np.uint8)
        per = O.sf_mma_bytes(cap, D // 16)
        for l in range(BH):
            for r in range(t0, t0 + n):
                for c in range(D // 16):
                    want[l * per + O.sf_mma_offset(r, c, D // 16)] = rs[l, r, c]
        assert np.array_equal(scales.cpu().numpy(), want)
    else:
        assert np.array_equal(scales.cpu().numpy(), rs.reshape(-1))


@pytest.mark.parametrize("name", SHAPES)
def test_transposed_columns_both_paths(name):
    g = torch.Generator().manual_seed(3)
    x = (torch.randn(2, 48, 40, generator=g) * torch.linspace(0.1, 10, 40)).to(torch.bfloat16)
    with path(name):
        c, sf, gs = nv.quantize_mma_t(x.cuda())
        torch.cuda.synchronize()
    rc, rsf, rg = O.quantize_mma_t(_host(x), dtype=1)
    assert gs.item() == rg
    assert np.array_equal(c.cpu().numpy().reshape(-1), rc.reshape(-1))
    assert np.array_equal(sf.cpu().numpy().reshape(-1), rsf.reshape(-1))


def test_policy_boundaries_and_defaults():
    """A launch of exactly a bound's thread count takes that shape, one thread less sends it on to the
    next one; the bytes are the same either way, and the policy call restores what it replaced."""
    default = nv.search_policy()
    assert 0 < default[0] <= default[1]
    x = torch.randn(64 * 16, generator=torch.Generator().manual_seed(1)).cuda()
    outs = []
    for bounds in ((64 * 16, 0), (64 * 16 - 1, 64 * 4), (0, 64 * 4 - 1)):   # 64 blocks, window [-2, 6]
        prev = nv.search_policy(*bounds)
        try:
            outs.append([t.cpu() for t in nv.quantize_ex(x, -2, 6)])
        finally:
            assert nv.search_policy(*prev) == bounds
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    assert nv.search_policy() == default
    with pytest.raises(nv.NVFP4Error):
        nv.search_policy(-2, 5)
    assert nv.search_policy() == default
