"""Pins for the oracle's FP4-attention softmax: the exp method and the quantized softmax numerators.

exp_ss (Cody-Waite reduction + degree-7 Taylor polynomial in FP32) is checked against float64 exp;
the softmax rows against numpy (max over the allowed keys, the float64 sum) and against quantizing the
exp_ss values block by block with the tensor scale fl(1/2688) through the pinned block quantizer."""
import numpy as np
import pytest

from oracle import oracle as O

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
