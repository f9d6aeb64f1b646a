"""Pins for the oracle's tensor-core consumer pieces: the 128x4 block-scale tile layout and the NVFP4
product D = alpha * g_a * g_b * A B^T.

The layout is NVIDIA's documented block-scaled MMA scale format (PTX ISA, tcgen05 block scaling;
cuBLAS "1D block scaling factors layout"): 512-byte tiles of 128 rows x 4 block columns, each tile a
[32][4][4] byte array indexed [row mod 32][row div 32][column].  The pins rebuild that array with
numpy reshapes (no offset formula), check documented offsets by hand, padding, and bijectivity.
The product is pinned against exact rational arithmetic and against a one-hot special case."""
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O


def _tiles_by_reshape(S: np.ndarray) -> np.ndarray:
    """[rows, bpr] with rows % 128 == 0 and bpr % 4 == 0 -> tile bytes, built from the [32][4][4] tile."""
    rows, bpr = S.shape
    RT, CT = rows // 128, bpr // 4
    # r = 128*rt + 32*j + i, c = 4*ct + cc  ->  tile (rt, ct), byte [i][j][cc]
    t = S.reshape(RT, 4, 32, CT, 4)            # (rt, j, i, ct, cc)
    t = t.transpose(0, 3, 2, 1, 4)             # (rt, ct, i, j, cc)
    return np.ascontiguousarray(t).reshape(-1)


@pytest.mark.parametrize("rows,bpr", [(128, 4), (256, 8), (384, 12), (128, 512)])
def test_layout_matches_tile_array_construction(rows, bpr):
    rng = np.random.default_rng(rows + bpr)
    S = rng.integers(1, 127, size=(rows, bpr), dtype=np.uint8)
    assert np.array_equal(O.scales_to_mma(S, 1, rows, bpr), _tiles_by_reshape(S))


def test_layout_documented_offsets():
    # inside the first tile: byte 16*(r mod 32) + 4*(r div 32) + c
    cases = {(0, 0): 0, (1, 0): 16, (31, 0): 496, (32, 0): 4, (64, 1): 9, (96, 3): 15, (127, 3): 511, (5, 2): 82}
    for (r, c), off in cases.items():
        assert O.sf_mma_offset(r, c, 8) == off, (r, c)
    # column tiles of one row tile are consecutive; then the next row tile
    assert O.sf_mma_offset(0, 4, 8) == 512
    assert O.sf_mma_offset(0, 4, 16) == 512
    assert O.sf_mma_offset(128, 0, 8) == 2 * 512
    assert O.sf_mma_offset(128, 0, 16) == 4 * 512
    assert O.sf_mma_offset(128, 0, 5) == 2 * 512     # 5 block columns pad to 2 column tiles


@pytest.mark.parametrize("rows,bpr", [(1, 1), (200, 6), (129, 4), (127, 9), (300, 2)])
def test_layout_ragged_bijective_with_zero_padding(rows, bpr):
    nbytes = O.sf_mma_bytes(rows, bpr)
    assert nbytes == -(-rows // 128) * -(-bpr // 4) * 512
    offs = [O.sf_mma_offset(r, c, bpr) for r in range(rows) for c in range(bpr)]
    assert len(set(offs)) == len(offs) and min(offs) >= 0 and max(offs) < nbytes
    rng = np.random.default_rng(rows * 7 + bpr)
    S = rng.integers(1, 127, size=(2, rows, bpr), dtype=np.uint8)
    out = O.scales_to_mma(S, 2, rows, bpr)
    assert out.size == 2 * nbytes
    for l in range(2):
        part = out[l * nbytes:(l + 1) * nbytes]
        used = np.zeros(nbytes, bool)
        used[offs] = True
        assert np.array_equal(part[offs], S[l].reshape(-1))
        assert not part[~used].any()                  # padding bytes are zero


def test_layout_padded_case_agrees_with_reshape_after_padding():
    rows, bpr = 200, 6
    rng = np.random.default_rng(3)
    S = rng.integers(1, 127, size=(rows, bpr), dtype=np.uint8)
    P = np.zeros((256, 8), np.uint8)
    P[:rows, :bpr] = S
    assert np.array_equal(O.scales_to_mma(S, 1, rows, bpr), _tiles_by_reshape(P))


def test_block_values_equal_dequantize_with_unit_tensor_scale():
    rng = np.random.default_rng(5)
    rows, cols = 8, 64
    x = rng.standard_normal(rows * cols).astype(np.float32)
    codes, scales, _, _, _ = O.quantize(x, -2, 6, gscale_in=1.0 / 64)
    # with g = 1 every product E2M1 * E4M3 is exact in FP32, so dequantize gives the real values
    ref = O.dequantize(codes, scales, 1.0).astype(np.float64).reshape(rows, cols)
    assert np.array_equal(O.block_values(codes, scales, rows, cols), ref)


def _exact_gemm(a_codes, a_scales, b_codes, b_scales, M, N, K):
    t2 = [Fraction(O.e2m1_decode(c)) for c in range(16)]
    t4 = [Fraction(O.e4m3_decode(c)) for c in range(127)]   # finite, non-negative scale codes

    def val(codes, scales, r, k):
        byte = int(codes[(r * K + k) // 2])
        q = (byte >> 4) if k % 2 else (byte & 15)
        return t2[q] * t4[int(scales[r * (K // 16) + k // 16])]

    return [[sum(val(a_codes, a_scales, i, k) * val(b_codes, b_scales, j, k) for k in range(K)) for j in range(N)]
            for i in range(M)]


def test_gemm_oracle_matches_exact_rational_sum():
    rng = np.random.default_rng(11)
    M, N, K = 3, 4, 48
    a = rng.integers(0, 256, size=M * K // 2, dtype=np.uint8)
    b = rng.integers(0, 256, size=N * K // 2, dtype=np.uint8)
    sa = rng.integers(20, 100, size=M * K // 16, dtype=np.uint8)
    sb = rng.integers(20, 100, size=N * K // 16, dtype=np.uint8)
    alpha, ga, gb = 0.75, 2.0 ** -3, 3.0
    got = O.gemm_nt(a, sa, ga, b, sb, gb, M, N, K, alpha)[0]
    ex = _exact_gemm(a, sa, b, sb, M, N, K)
    for i in range(M):
        for j in range(N):
            want = float(ex[i][j] * Fraction(alpha) * Fraction(ga) * Fraction(gb))
            assert got[i, j] == want, (i, j, got[i, j], want)


def test_gemm_oracle_one_hot_b_selects_a_column():
    rng = np.random.default_rng(12)
    M, N, K = 5, 3, 32
    x = rng.standard_normal(M * K).astype(np.float32)
    a_codes, a_scales, ga, _, _ = O.quantize(x, -2, 6)
    av = O.block_values(a_codes, a_scales, M, K)
    cols = [0, 17, 31]
    b_codes = np.zeros(N * K // 2, np.uint8)
    b_scales = np.full(N * K // 16, 56, np.uint8)          # E4M3 code 56 = 1.0
    for n, k in enumerate(cols):
        b_codes[(n * K + k) // 2] |= np.uint8(2 << (4 * (k % 2)))   # E2M1 code 2 = 1.0
    d = O.gemm_nt(a_codes, a_scales, ga, b_codes, b_scales, 1.0, M, N, K, alpha=2.0)[0]
    for n, k in enumerate(cols):
        assert np.array_equal(d[:, n], 2.0 * float(ga) * av[:, k])


def test_quantize_mma_is_quantize_plus_layout():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((2, 130, 96)).astype(np.float32)
    codes, sf, g = O.quantize_mma(x)
    c2, s2, g2, _, _ = O.quantize(x.reshape(-1))
    assert g == g2 and np.array_equal(codes, c2)
    assert np.array_equal(sf, O.scales_to_mma(s2, 2, 130, 6))
