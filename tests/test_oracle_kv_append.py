"""Pins for the oracle's incremental KV append (decode-time growth of the NVFP4 middle of the cache).

Given the tensor scale, blocks are independent, so appending the middle tokens group by group must
reproduce the one-shot mixed-precision layout computed with the same scale, and one appended token
must equal its rotated row groups quantized on their own."""
import numpy as np
import pytest
import torch

from nvfp4_block_scaled_11_b200 import workloads as W
from oracle import oracle as O


def _k16(T, heads=2):
    k = W.kv_bf16("cpu", scale=T / 32768, heads=heads)
    return k.view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("T,group", [(100, 16), (77, 16), (64, 1), (150, 7)])
def test_grouped_append_reproduces_one_shot_layout(T, group):
    k = _k16(T)
    B, H, T, D = k.shape
    _, _, c, s, g = O.kv_mixed(k)
    Tm = T - 32
    cap = Tm + 40
    cc = np.zeros((B * H, cap, D // 2), np.uint8)
    ss = np.zeros((B * H, cap, D // 16), np.uint8)
    t = 0
    while t < Tm:
        n = min(group, Tm - t)
        O.kv_append(k.reshape(B * H, T, D), 16 + t, n, g, cc, ss, t)
        t += n
    assert np.array_equal(cc[:, :Tm], c.reshape(B * H, Tm, D // 2))
    assert np.array_equal(ss[:, :Tm], s.reshape(B * H, Tm, D // 16))
    assert not cc[:, Tm:].any() and not ss[:, Tm:].any()


def test_single_token_equals_rotated_blocks_quantized_alone():
    k = _k16(40, heads=1)
    T, D = k.shape[2], k.shape[3]
    rows = k.reshape(1, T, D)
    g = np.float32(0.0021)
    cap, t0, tok = 8, 5, 23
    cc = np.full((1, cap, D // 2), 0xAA, np.uint8)
    ss = np.full((1, cap, D // 16), 0xAA, np.uint8)
    O.kv_append(rows, tok, 1, g, cc, ss, t0)
    rot = O.hadamard16(rows[0, tok].copy(), dtype=O.BF16, out_dtype=O.F32)
    rc, rs, _, _ = O.quantize_blocks(rot, 0, D // 16, g)
    assert np.array_equal(cc[0, t0], rc) and np.array_equal(ss[0, t0], rs)
    others = [r for r in range(cap) if r != t0]
    assert (cc[0, others] == 0xAA).all() and (ss[0, others] == 0xAA).all()   # untouched rows


def test_unrotated_append_and_capacity_errors():
    D = 64
    k = _k16(36, heads=1)[..., :D].copy()
    T = k.shape[2]
    rows = k.reshape(1, T, D)
    g = np.float32(0.003)
    cc = np.zeros((1, 4, D // 2), np.uint8)
    ss = np.zeros((1, 4, D // 16), np.uint8)
    O.kv_append(rows, 10, 4, g, cc, ss, 0, rotate=0)
    x = np.ascontiguousarray(rows[0, 10:14]).reshape(-1)
    rc, rs, _, _ = O.quantize_blocks(x, 0, x.size // 16, g, dtype=O.BF16)
    assert np.array_equal(cc.reshape(-1), rc) and np.array_equal(ss.reshape(-1), rs)
    with pytest.raises(ValueError):
        O.kv_append(rows, 0, 3, g, cc, ss, 2)      # rows 2..4 exceed the 4-row cache
