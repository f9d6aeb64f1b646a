"""Pins for the oracle's FP4-attention softmax: the exp method and the quantized softmax numerators.

exp_ss (Cody-Waite reduction + degree-7 Taylor polynomial in FP32) is checked against float64 exp;
the softmax rows against numpy (max over the allowed keys, the float64 sum) and against quantizing the
exp_ss values block by block with the tensor scale fl(1/2688) through the pinned block quantizer."""
import math
import os
import sys
from fractions import Fraction

import numpy as np
import pytest

from oracle import oracle as O

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))
import exact_f32 as X  # noqa: E402

U = 2.0 ** -24


def test_exp_ss_accuracy_and_special_values():
    rng = np.random.default_rng(0)
    xs = np.float32(-rng.uniform(0, 87, 20000))
    got = np.array([O.exp_ss(x) for x in xs], np.float64)
    ref = np.exp(xs.astype(np.float64))
    assert (np.abs(got - ref) <= 2 * U * ref).all()                 # normal results: within 2 ulp
    sub = np.float32(-rng.uniform(87.5, 103.9, 2000))
    got2 = np.array([O.exp_ss(x) for x in sub], np.float64)
    assert (np.abs(got2 - np.exp(sub.astype(np.float64))) <= 2.0 ** -149).all()   # subnormal results
    assert O.exp_ss(0.0) == 1.0 and O.exp_ss(-0.0) == 1.0
    assert O.exp_ss(-104.5) == 0.0 and O.exp_ss(-np.inf) == 0.0
    assert np.isnan(O.exp_ss(np.nan))
    sweep = np.float32(np.linspace(-30, 0, 5001))
    vals = np.array([O.exp_ss(x) for x in sweep])
    assert (np.diff(vals) >= 0).all()                                  # monotone


def _scores(batch, Tq, Tk, seed, scale=3.0):
    return (np.random.default_rng(seed).standard_normal((batch, Tq, Tk)) * scale).astype(np.float32)


@pytest.mark.parametrize("causal,q_offset", [(False, 0), (True, 0), (True, 17)])
def test_softmax_quantize_rows(causal, q_offset):
    batch, Tq, Tk = 2, 5, 64
    s = _scores(batch, Tq, Tk, 1)
    codes, scales, m, l, g = O.softmax_quantize(s, causal, q_offset)
    assert g == np.float32(1.0) / np.float32(2688.0)
    for b in range(batch):
        for q in range(Tq):
            allowed = np.arange(Tk) <= q + q_offset if causal else np.ones(Tk, bool)
            assert m[b, q] == s[b, q][allowed].max()
            e64 = np.where(allowed, np.exp(s[b, q].astype(np.float64) - float(m[b, q])), 0.0)
            assert abs(float(l[b, q]) - e64.sum()) <= (Tk + 4) * U * e64.sum()
            # the quantized row equals the block quantizer on the exp_ss values
            ev = np.array([O.exp_ss(s[b, q, k] - m[b, q]) if allowed[k] else 0.0 for k in range(Tk)], np.float32)
            rc, rs, _, _ = O.quantize_blocks(ev, 0, Tk // 16, g)
            assert np.array_equal(codes[b, q], rc) and np.array_equal(scales[b, q], rs)
            # masked keys decode to zero
            q4 = np.empty(Tk, np.uint8)
            q4[0::2], q4[1::2] = codes[b, q] & 15, codes[b, q] >> 4
            assert not (q4[~allowed] & 7).any()


def test_softmax_quantize_rejects_ragged_keys():
    with pytest.raises(ValueError):
        O.softmax_quantize(np.zeros((1, 2, 24), np.float32))


# ln 2 to 60 digits (a mathematical constant; the method's constants are derived from it below)
LN2 = Fraction("0.693147180559945309417232121458176568075500134360255254120680009")


def _round_sig(q: Fraction, bits: int) -> Fraction:
    """q > 0 rounded to nearest with `bits` significant bits."""
    e = q.numerator.bit_length() - q.denominator.bit_length()
    while Fraction(2) ** e > q:
        e -= 1
    while Fraction(2) ** (e + 1) <= q:
        e += 1
    quantum = Fraction(2) ** (e - bits + 1)
    return X.rint_even(q / quantum) * quantum


def _exp_exact_route(x: float) -> np.float32:
    """The Cody-Waite + Taylor-7 method evaluated on exact rationals, each operation rounded once to
    binary32 by the software rounding of tests/exact_f32.py: t = fl(x log2e), n = rint(t),
    r = fma(n, -ln2_lo, fma(n, -ln2_hi, x)), Horner with fused multiply-adds over 1/7!, ..., 1/2!, 1, 1,
    then p * 2^n rounded once.  The constants are derived here from ln 2 and the factorials."""
    log2e = X.rne(1 / LN2)
    ln2_hi = _round_sig(LN2, 16)
    ln2_lo = X.rne(LN2 - ln2_hi)
    coef = [X.rne(Fraction(1, math.factorial(k))) for k in range(7, 1, -1)] + [Fraction(1), Fraction(1)]
    xq = X.f(x)
    n = X.rint_even(X.mul(xq, log2e))
    r = X.fma(Fraction(n), -ln2_lo, X.fma(Fraction(n), -ln2_hi, xq))
    p = coef[0]
    for c in coef[1:]:
        p = X.fma(p, r, c)
    return X.to_f32(p * Fraction(2) ** n)


def test_exp_ss_bits_equal_an_exact_evaluation_of_the_method():
    """Pins the exact bits of exp_ss (which decide P~'s codes): every result equals the same published
    method evaluated through exact rational arithmetic with one binary32 rounding per operation, on a
    dense grid of [-104, 0] (random points, the points where x log2e crosses a half-integer, the
    subnormal-result range and the ends)."""
    rng = np.random.default_rng(7)
    pts = [np.float32(-rng.uniform(0, 104, 3000)),
           np.float32(-rng.uniform(86, 104, 1500)),                 # subnormal and smallest normal results
           np.float32(-rng.uniform(0, 1e-3, 200))]
    # x near (j + 1/2) ln 2: the reduction's integer n changes there
    half = np.array([(j + 0.5) * 0.6931471805599453 for j in range(0, 151)])
    c = np.float32(-half)
    near = np.concatenate([c, np.nextafter(c, np.float32(-np.inf)), np.nextafter(c, np.float32(np.inf))])
    pts.append(near.astype(np.float32))
    pts.append(np.float32([0.0, -0.0, -1e-30, -104.0, np.nextafter(np.float32(-104), np.float32(0))]))
    xs = np.concatenate(pts)
    xs = xs[(xs >= -104) & (xs <= 0)]
    bad = [(float(x), float(O.exp_ss(x)), float(_exp_exact_route(x))) for x in xs
           if O.exp_ss(x).view(np.uint32) != _exp_exact_route(x).view(np.uint32)]
    assert not bad, bad[:5]


def test_exact_rounding_helper_against_numpy_casts():
    """The software rounding used above agrees with numpy's float64 -> float32 cast (round to nearest even,
    gradual underflow), ties included."""
    rng = np.random.default_rng(3)
    vals = np.concatenate([rng.standard_normal(3000) * 10.0 ** rng.integers(-44, 38, 3000),
                           rng.uniform(-1e-44, 1e-44, 500)])
    ties = [1 + 2.0 ** -24, 1 + 3 * 2.0 ** -24, 2.0 ** -149 * 1.5, 2.0 ** -149 * 2.5, -(1 + 2.0 ** -24)]
    for v in list(vals) + ties:
        assert X.to_f32(Fraction(float(v))) == np.float32(v) or np.isinf(np.float32(v))
