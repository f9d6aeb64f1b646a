"""Incremental KV cache (decode) through the C ABI against the oracle: bit-exact codes and scales."""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_11_b200 as nv
from nvfp4_block_scaled_11_b200 import workloads as W
from nvfp4_block_scaled_11_b200.kvcache import NVFP4KVCache
from oracle import oracle as O

pytestmark = pytest.mark.gpu


def _u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _k(T, heads=2, D=128):
    k = W.kv_bf16("cpu", scale=T / 32768, heads=heads, head_dim=D)
    return k


@pytest.mark.parametrize("rotate", [True, False])
@pytest.mark.parametrize("tile", [False, True])
def test_kv_append_matches_oracle(rotate, tile):
    k = _k(64, heads=3)[0]                      # [BH=3, T, D]
    BH, T, D = k.shape
    first, n, cap, t0 = 7, 20, 300, 131         # rows 131..150 cross a 128-row tile boundary
    g = torch.tensor([0.0023], dtype=torch.float32)
    codes = torch.full((BH, cap, D // 2), 0xAA, dtype=torch.uint8, device="cuda")
    if tile:
        scales = torch.full((nv.sf_mma_bytes(cap, D, BH),), 0xAA, dtype=torch.uint8, device="cuda")
    else:
        scales = torch.full((BH, cap, D // 16), 0xAA, dtype=torch.uint8, device="cuda")
    nv.kv_append(k.cuda(), first, n, g.cuda(), codes, scales, t0, rotate=rotate, tile_layout=tile)
    rc = np.full((BH, cap, D // 2), 0xAA, np.uint8)
    rs = np.full((BH, cap, D // 16), 0xAA, np.uint8)
    O.kv_append(_u16(k), first, n, g.item(), rc, rs, t0, rotate=int(rotate))
    assert np.array_equal(codes.cpu().numpy(), rc)
    if not tile:
        assert np.array_equal(scales.cpu().numpy(), rs)
    else:
        want = np.full(nv.sf_mma_bytes(cap, D, BH), 0xAA, np.uint8)
        per = O.sf_mma_bytes(cap, D // 16)
        for l in range(BH):
            for r in range(t0, t0 + n):
                for c in range(D // 16):
                    want[l * per + O.sf_mma_offset(r, c, D // 16)] = rs[l, r, c]
        assert np.array_equal(scales.cpu().numpy(), want)


def test_kv_gscale_matches_kv_mixed():
    k = _k(200)
    g = nv.kv_gscale(k.cuda())
    *_, rg = O.kv_mixed(_u16(k))
    assert g.item() == rg
    g0 = nv.kv_gscale(k.cuda(), rotate=False)
    *_, rg0 = O.kv_mixed(_u16(k), rotate=0)
    assert g0.item() == rg0


def test_kv_append_errors():
    k = torch.zeros((2, 32, 64), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(1, device="cuda")
    codes = torch.zeros((2, 8, 32), dtype=torch.uint8, device="cuda")
    scales = torch.zeros((2, 8, 4), dtype=torch.uint8, device="cuda")
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_append(k, 0, 5, g, codes, scales, 4)        # rows 4..8 exceed the 8-row cache
    assert e.value.status == -2
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_append(k, 30, 4, g, codes, scales, 0)       # tokens 30..33 exceed T = 32
    assert e.value.status == -2
    nv.kv_append(k, 0, 0, g, codes, scales, 8)             # nothing to do


@pytest.mark.parametrize("tile", [False, True])
def test_decode_cache_matches_oracle_sequence(tile):
    B, H, D, T0 = 1, 2, 128, 90
    full = _k(T0 + 60, heads=H)                  # the whole sequence: prefill + decoded tokens
    Tfull = full.shape[2]
    pre = full[:, :, :T0].contiguous()
    cache = NVFP4KVCache(B, H, D, capacity=256, tile_layout=tile)
    cache.prefill(pre.cuda())
    t = T0
    for _ in range(37):                          # one token per step
        cache.append(full[:, :, t:t + 1].cuda())
        t += 1
    cache.append(full[:, :, t:Tfull].cuda())     # then a chunk
    torch.cuda.synchronize()
    assert cache.length == Tfull
    # oracle: g from the prefill, the middle = tokens [16, 16 + n_mid) of the whole sequence
    *_, g = O.kv_mixed(_u16(pre))
    assert cache.gscale.item() == g
    n_mid = cache.n_mid
    assert n_mid == Tfull - 16 - cache.n_window and cache.recent <= cache.n_window < 2 * cache.recent
    rc = np.zeros((B * H, 256, D // 2), np.uint8)
    rs = np.zeros((B * H, 256, D // 16), np.uint8)
    O.kv_append(_u16(full).reshape(B * H, Tfull, D), 16, n_mid, g, rc, rs, 0)
    assert np.array_equal(cache.codes.cpu().numpy().reshape(B * H, 256, D // 2)[:, :n_mid], rc[:, :n_mid])
    if tile:
        assert np.array_equal(cache.scales.cpu().numpy(), O.scales_to_mma(rs, B * H, 256, D // 16))
    else:
        assert np.array_equal(cache.scales.cpu().numpy().reshape(B * H, 256, D // 16)[:, :n_mid], rs[:, :n_mid])
    assert torch.equal(cache.sink.cpu(), full[:, :, :16])
    assert torch.equal(cache.recent_tokens().cpu(), full[:, :, Tfull - cache.n_window:])


def _append_item(k, first, n, g, cap, t0, rotate, tile):
    """Device buffers (prefilled with 0xAA) and the oracle's expected bytes for one KV append."""
    BH, T, D = k.shape
    codes = torch.full((BH, cap, D // 2), 0xAA, dtype=torch.uint8, device="cuda")
    nsf = nv.sf_mma_bytes(cap, D, BH) if tile else BH * cap * (D // 16)
    scales = torch.full((nsf,), 0xAA, dtype=torch.uint8, device="cuda")
    rc = np.full((BH, cap, D // 2), 0xAA, np.uint8)
    rs = np.full((BH, cap, D // 16), 0xAA, np.uint8)
    O.kv_append(_u16(k), first, n, g, rc, rs, t0, rotate=int(rotate))
    if tile:
        want = np.full(nsf, 0xAA, np.uint8)
        per = O.sf_mma_bytes(cap, D // 16)
        for l in range(BH):
            for r in range(t0, t0 + n):
                for c in range(D // 16):
                    want[l * per + O.sf_mma_offset(r, c, D // 16)] = rs[l, r, c]
    else:
        want = rs.reshape(-1)
    item = (k.cuda(), first, n, torch.tensor([g], dtype=torch.float32, device="cuda"), codes, scales, t0, rotate, tile)
    return item, rc, want


@pytest.mark.parametrize("policy", [None, (0, None)])     # small batch: 16 lanes per block; or 4 x 3
def test_kv_append_batch_matches_oracle(policy):
    """Heterogeneous items (heads, head_dim, rotation, scale layout, rows, tensor scale) in one launch:
    each item's bytes equal the oracle's kv_append; an empty item is skipped."""
    specs = [(3, 64, 128, True, False, 5, 16, 100, 7, 0.0021), (2, 40, 64, True, True, 0, 16, 300, 120, 0.0033),
             (1, 33, 128, False, False, 17, 16, 64, 48, 0.0017), (4, 20, 32, False, True, 2, 3, 130, 127, 0.004),
             (2, 16, 128, True, False, 0, 0, 16, 16, 0.002)]
    items, want = [], []
    for i, (BH, T, D, rot, tile, first, n, cap, t0, g) in enumerate(specs):
        k = W.kv_decode_keys("cpu", n=T, heads=BH, head_dim=D) * (1.0 + i)
        item, rc, rs = _append_item(k.to(torch.bfloat16), first, n, g, cap, t0, rot, tile)
        items.append(item)
        want.append((rc, rs))
    prev = nv.search_policy(*policy) if policy else None
    try:
        nv.kv_append_batch(items)
        torch.cuda.synchronize()
    finally:
        if prev:
            nv.search_policy(*prev)
    for item, (rc, rs) in zip(items, want):
        assert np.array_equal(item[4].cpu().numpy(), rc)
        assert np.array_equal(item[5].cpu().numpy(), rs)


def test_kv_append_batch_errors_launch_nothing():
    k = W.kv_decode_keys("cpu", n=32, heads=2, head_dim=64)
    good, _, _ = _append_item(k, 0, 16, 0.002, 64, 0, True, False)
    bad = (good[0], 0, 16, good[3], good[4], good[5], 60, True, False)       # rows 60..75 exceed cap 64
    before = good[4].clone()
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_append_batch([good, bad])
    assert e.value.status == -2
    with pytest.raises(nv.NVFP4Error) as e:
        nv.kv_append_batch([good], -16, 16)                                     # 33 offsets
    assert e.value.status == -1
    with pytest.raises(ValueError):
        nv.kv_append_batch([good] * 65)
    torch.cuda.synchronize()
    assert torch.equal(good[4], before)                                         # nothing was launched
    nv.kv_append_batch([])


@pytest.mark.parametrize("tile", [False, True])
def test_cache_group_equals_separate_appends(tile):
    """Several caches (the K and V of three layers, different head counts, rotated or not) stepped
    together -- through a persistent NVFP4KVCacheGroup, and through append_many -- with one batched flush
    per step give the same state as appending to each cache on its own; a cache whose window is not full
    is skipped within the batch (one layer starts a token later)."""
    from nvfp4_block_scaled_11_b200.kvcache import NVFP4KVCacheGroup, append_many
    B, D, T0, steps = 1, 128, 40, 45
    shapes = [2, 2, 3, 3, 1, 1]
    ahead = [0, 0, 1, 1, 0, 0]                   # layer 1's windows hold one more token: they fill earlier
    seqs = [W.kv_decode_keys("cpu", n=T0 + 1 + steps, heads=h, head_dim=D)[None] * (1 + 0.5 * i)
            for i, h in enumerate(shapes)]
    seqs = [s.to(torch.bfloat16) for s in seqs]

    def make():
        cs = [NVFP4KVCache(B, h, D, capacity=128, tile_layout=tile, rotate=(i % 2 == 0))
              for i, h in enumerate(shapes)]
        for c, s, ah in zip(cs, seqs, ahead):
            c.prefill(s[:, :, :T0].cuda())
            if ah:
                c.append(s[:, :, T0:T0 + ah].cuda())
        return cs

    a, b, c3 = make(), make(), make()
    group = NVFP4KVCacheGroup(a)
    for step in range(steps):
        rows = [s[:, :, T0 + ah + step:T0 + ah + step + 1].cuda() for s, ah in zip(seqs, ahead)]
        group.append(rows)
        append_many(c3, rows)
        for c, r in zip(b, rows):
            c.append(r)
    torch.cuda.synchronize()
    for c1, c2, c4 in zip(a, b, c3):
        for c in (c1, c4):
            assert (c.n_mid, c.n_window, c.head) == (c2.n_mid, c2.n_window, c2.head) and c.n_mid > 16
            assert torch.equal(c.codes, c2.codes) and torch.equal(c.scales, c2.scales)
            assert torch.equal(c.window, c2.window)
