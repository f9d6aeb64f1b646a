"""Pins for the oracle's MXFP4 (OCP MX v1.0: 32-element blocks, E8M0 scale 2^(floor(log2 amax) - 2),
E2M1 elements with round-to-nearest-even and saturation).

The expected values come by another route: the block exponent from numpy's frexp (not the oracle's
bit manipulation), the element rounding from ml_dtypes' float4_e2m1fn cast (not the oracle's
converter), and scale values from ml_dtypes' float8_e8m0fnu."""
import ml_dtypes
import numpy as np
import pytest
import torch

from oracle import oracle as O


def _expected(x32: np.ndarray):
    blocks = x32.reshape(-1, 32)
    amax = np.abs(blocks).max(axis=1)
    _, ex = np.frexp(amax.astype(np.float64))          # amax = m * 2^ex, m in [0.5, 1)
    e = np.where(amax == 0, -127, np.clip(ex - 1 - 2, -127, 127)).astype(np.int64)
    inv = np.ldexp(np.float32(1.0), -e).astype(np.float32)  # exact powers of two
    y = (blocks * inv[:, None]).astype(np.float32)
    q = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    codes = (q[:, 0::2] | (q[:, 1::2] << 4)).astype(np.uint8).reshape(-1)
    return codes, (e + 127).astype(np.uint8)


@pytest.mark.parametrize("kind", ["normal", "student", "tiny", "huge", "mixed_scale"])
def test_mxfp4_quantize_matches_library_casts(kind):
    rng = np.random.default_rng(hash(kind) % 2 ** 32)
    n = 32 * 512
    if kind == "normal":
        x = rng.standard_normal(n)
    elif kind == "student":
        x = rng.standard_t(3, n)
    elif kind == "tiny":
        x = rng.standard_normal(n) * 1e-39          # subnormal magnitudes
    elif kind == "huge":
        x = rng.standard_normal(n) * 1e37
    else:
        x = rng.standard_normal(n) * np.repeat(10.0 ** rng.uniform(-20, 20, n // 32), 32)
    x = x.astype(np.float32)
    x[:32] = 0.0
    x[32:64] = -0.0 * x[32:64]
    codes, scales = O.mxfp4_quantize(x)
    ec, es = _expected(x)
    assert np.array_equal(scales, es)
    assert np.array_equal(codes, ec)


def test_mxfp4_dequantize_matches_library_decode():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal(32 * 64) * 3).astype(np.float32)
    codes, scales = O.mxfp4_quantize(x)
    got = O.mxfp4_dequantize(codes, scales)
    q = np.empty(x.size, np.uint8)
    q[0::2], q[1::2] = codes & 15, codes >> 4
    v = q.view(ml_dtypes.float4_e2m1fn).astype(np.float32)
    X = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float32)
    assert np.array_equal(got, v * np.repeat(X, 32))


def test_mxfp4_special_blocks_and_saturation():
    x = np.zeros(32 * 4, np.float32)
    x[0:32] = -0.0                                   # zero block: scale byte 0, sign-only codes
    x[32:64] = np.linspace(-1, 1, 32)
    x[40] = np.nan                                   # NaN block
    x[64:96] = 1.0
    x[70] = np.inf                                   # Inf block
    x[96:128] = 0.5
    x[100] = 7.9 * 2.0 ** 5                          # y = 7.9 saturates to 6
    codes, scales = O.mxfp4_quantize(x)
    assert scales[0] == 0 and (codes[:16] == 0x88).all()
    assert scales[1] == 0xFF and not codes[16:32].any()
    assert scales[2] == 0xFF and not codes[32:48].any()
    assert scales[3] == 127 + 5 and (codes[48 + 2] & 15) == 7   # code 7 = 6.0
    d = O.mxfp4_dequantize(codes, scales)
    assert np.isnan(d[32:96]).all() and d[100] == 6.0 * 32


def test_mxfp4_round_trip_of_representable_blocks():
    rng = np.random.default_rng(9)
    vals = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    x = np.empty(32 * 100, np.float32)
    for b in range(100):
        k = int(rng.integers(-100, 100))
        v = rng.choice(vals, 32) * rng.choice([-1, 1], 32)
        v[rng.integers(32)] = rng.choice([4.0, 6.0])   # block max in [4, 8): exponent e = k
        x[32 * b:32 * b + 32] = (v * 2.0 ** k).astype(np.float32)
    codes, scales = O.mxfp4_quantize(x)
    assert np.array_equal(O.mxfp4_dequantize(codes, scales), x)


def test_mxfp4_bf16_input():
    t = torch.randn(32 * 32).to(torch.bfloat16)
    u16 = t.view(torch.int16).numpy().view(np.uint16)
    c1, s1 = O.mxfp4_quantize(u16, O.BF16)
    c2, s2 = O.mxfp4_quantize(t.float().numpy())
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
