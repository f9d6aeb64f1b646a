"""Pins of the oracle's ScaleSearch, dequantize, Hadamard-16 and KV layout against things other than
itself: an independent brute-force search over every E4M3 code (numpy + ml_dtypes), closed forms
(exactly representable blocks), invariants of the method, and library matrix products."""
import math

import ml_dtypes as md
import numpy as np
import pytest

from oracle import oracle as O
from tests import brute

RNG = np.random.default_rng(1234)


def _blocks(kind, nb, rng):
    if kind == "normal":
        return rng.standard_normal((nb, 16)).astype(np.float32)
    if kind == "student":
        z = rng.standard_normal((nb, 16))
        chi = (rng.standard_normal((nb, 16, 3)) ** 2).sum(-1) / 3
        return (0.5 * z / np.sqrt(chi)).astype(np.float32)
    if kind == "outlier":
        x = rng.standard_normal((nb, 16))
        x[np.arange(nb), rng.integers(0, 16, nb)] *= 30
        return x.astype(np.float32)
    if kind == "uniform":
        return rng.uniform(-1, 1, (nb, 16)).astype(np.float32)
    if kind == "lognormal":
        return (rng.lognormal(0, 2, (nb, 16)) * rng.choice([-1, 1], (nb, 16))).astype(np.float32)
    if kind == "grid":  # values on or next to E2M1 decision points relative to a unit scale
        pts = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
        x = rng.choice(pts, (nb, 16)) * rng.choice([-1, 1], (nb, 16))
        x = x * np.float32(2.0) ** rng.integers(-3, 3, (nb, 1))
        nudge = rng.choice([0, 1, -1], (nb, 16))
        return np.nextafter(x.astype(np.float32), np.where(nudge > 0, np.inf, -np.inf).astype(np.float32)) * (nudge != 0) + x * (nudge == 0)
    raise KeyError(kind)


def _search_all(X, g, f_lo, f_hi):
    res = [O.search_block(X[b], g, f_lo, f_hi) for b in range(X.shape[0])]
    codes = np.stack([r[0] for r in res])
    sc = np.array([r[1] for r in res])
    fs = np.array([r[2] for r in res])
    sse = np.array([r[3] for r in res], np.float32)
    return codes, sc, fs, sse


@pytest.mark.parametrize("kind", ["normal", "student", "outlier", "uniform", "lognormal", "grid"])
@pytest.mark.parametrize("window", [(-2, 6), (0, 0), (-8, 8)])
def test_search_matches_brute_force(kind, window):
    """I3: the oracle's f* and SSE equal the argmin over the window of an exhaustive score of every code."""
    X = _blocks(kind, 96, RNG).astype(np.float32)
    X = X.astype(np.float32)
    g = np.float32(np.abs(X).max() / np.float32(2688.0))
    f_lo, f_hi = window
    bf, bs, c0, tab = brute.search(X, g, f_lo, f_hi)
    codes, sc, fs, sse = _search_all(X, g, f_lo, f_hi)
    assert np.array_equal(fs, bf)
    ok = bf != -128
    assert np.array_equal(sse[ok].view(np.uint32), bs[ok].view(np.uint32))
    assert np.array_equal(sc[ok], (c0 + bf)[ok])
    # the codes are the library E2M1 cast of x * (1 / d*) with d* = dec(scale) * g
    for b in np.nonzero(ok)[0]:
        d = np.float32(brute.E4M3_VALUE[sc[b]] * g)
        r = np.float32(np.float32(1) / d)
        q = np.clip(X[b] * r, -6, 6).astype(md.float4_e2m1fn).view(np.uint8)
        assert np.array_equal(codes[b], (q[0::2] | (q[1::2] << 4)).astype(np.uint8))


def test_out_of_window_optimum_rate_is_reported():
    """The window [-2,6] is a restriction: the global optimum over all codes sometimes lies outside."""
    X = _blocks("normal", 512, RNG)
    g = np.float32(np.abs(X).max() / np.float32(2688.0))
    bf, bs, c0, tab = brute.search(X, g, -2, 6)
    glob = tab.min(1)
    outside = np.mean(glob < bs)
    assert 0.0 <= outside < 0.2  # rare on Gaussian blocks


def test_f0_window_equals_separate_max_scaling():
    """I1: the search restricted to f = 0 reproduces max-scaling (written separately)."""
    for kind in ("normal", "outlier", "lognormal", "grid"):
        X = _blocks(kind, 200, RNG)
        g = np.float32(np.abs(X).max() / np.float32(2688.0))
        for b in range(X.shape[0]):
            c1, s1, f1, e1 = O.search_block(X[b], g, 0, 0)
            c2, s2, e2 = O.maxscale_block(X[b], g)
            assert np.array_equal(c1, c2) and s1 == s2 and np.float32(e1).tobytes() == np.float32(e2).tobytes()
            assert f1 in (0, -128)


def test_exactly_representable_blocks_round_trip():
    """I2: with g = 1 (tensor amax 2688), blocks x = v * s with s an E4M3 value and v an E2M1 value, one
    element equal to 6 s, quantize with SSE 0, f* = 0 and dequantize back bit-exactly."""
    e2m1 = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    e4m3 = np.arange(1, 127, dtype=np.uint8).view(md.float8_e4m3fn).astype(np.float32)
    rows = [np.full(16, 2688.0, np.float32)]  # sets the tensor amax
    for s in e4m3:
        if 6 * s > 2688:
            continue
        v = RNG.choice(e2m1, 16) * RNG.choice([-1, 1], 16)
        v[RNG.integers(16)] = 6.0 * RNG.choice([-1, 1])
        rows.append((v * s).astype(np.float32))
    X = np.stack(rows).astype(np.float32)
    codes, scales, g, bf, bs = O.quantize(X.reshape(-1), -2, 6)
    assert g == np.float32(1.0)
    assert np.all(bf == 0) and np.all(bs == 0)
    back = O.dequantize(codes, scales, g)
    assert np.array_equal(back.view(np.uint32), X.reshape(-1).view(np.uint32))
    # signed zeros: -0.0 elements come back as -0.0
    assert np.array_equal(np.signbit(back), np.signbit(X.reshape(-1)))


def test_search_never_worse_than_max_scaling():
    """I6: for every block where f = 0 is a valid candidate, the search SSE <= the f = 0 SSE."""
    X = np.concatenate([_blocks(k, 300, RNG) for k in ("normal", "student", "outlier", "lognormal")])
    _, _, g, bf, bs = O.quantize(X.reshape(-1), -2, 6)
    _, _, g0, bf0, bs0 = O.quantize(X.reshape(-1), 0, 0)
    ok = bf0 == 0
    assert np.all(bs[ok] <= bs0[ok])
    assert bs.astype(np.float64).sum() < bs0.astype(np.float64).sum()


def test_bimodal_offsets_on_gaussian_blocks():
    """I4 (qualitative): the chosen offsets split between mapping amax to 6 (f near 0) and to 4
    (a scale about 1.5x larger, f near +4), with a dip in between; blocks in the second mode encode
    their largest element as 4 (magnitude code 0x6).  The exact histogram is not given on the page."""
    rng = np.random.default_rng(7)
    X = rng.standard_normal(1 << 18).astype(np.float32)
    codes, scales, g, bf, bs = O.quantize(X, -2, 6)
    hist = np.array([(bf == f).mean() for f in range(-2, 7)])
    low = hist[:4].max()          # f in [-2, 1]
    high = hist[5:].max()         # f in [3, 6]
    dip = hist[4]                 # f = 2
    assert low > 4 * dip and high > 4 * dip
    assert np.argmax(hist[:4]) in (1, 2) and np.argmax(hist[5:]) in (1, 2)
    sel = np.nonzero(bf >= 3)[0][:2000]
    Xb = X.reshape(-1, 16)
    for b in sel:
        imax = np.argmax(np.abs(Xb[b]))
        byte = codes[8 * b + imax // 2]
        nib = (byte >> 4) if imax & 1 else (byte & 0xF)
        assert nib & 7 == 6


def test_special_blocks():
    g = np.float32(1.0)
    # all zero (with -0.0): scale 0, sign-only codes, f = -128, sse 0
    z = np.zeros(16, np.float32)
    z[3] = -0.0
    c, s, f, e = O.search_block(z, g, -2, 6)
    assert s == 0 and f == -128 and e == 0
    assert (c[1] >> 4) == 0x8 and c[0] == 0
    # non-finite element: poisoned block
    for bad in (np.nan, np.inf, -np.inf):
        x = np.ones(16, np.float32)
        x[5] = bad
        c, s, f, e = O.search_block(x, g, -2, 6)
        assert s == 0x7F and f == -128 and np.all(c == 0) and np.isnan(e)
    # g NaN / inf / negative: poisoned
    for gg in (np.nan, np.inf, -1.0):
        c, s, f, e = O.search_block(np.ones(16, np.float32), np.float32(gg), -2, 6)
        assert s == 0x7F
    # g = 0 with a nonzero block: every candidate has d = 0 -> no valid candidate
    x = np.linspace(-1, 1, 16).astype(np.float32)
    c, s, f, e = O.search_block(x, np.float32(0.0), -2, 6)
    assert s == 0 and f == -128
    assert e == np.float32(sum(np.float64(v) ** 2 for v in x)) or abs(e - np.sum(x.astype(np.float64) ** 2)) < 1e-6
    # default code underflows to 0 and the window is {0}: no valid candidate
    x = np.full(16, 1e-6, np.float32)
    c, s, f, e = O.search_block(x, np.float32(1.0), 0, 0)
    assert s == 0 and f == -128
    # ... but positive offsets reach the subnormal scale codes
    c, s, f, e = O.search_block(x, np.float32(1e-6), 0, 3)
    assert s >= 1
    # saturated default code (block amax / 6 / g >= 448)
    x = np.full(16, 1000.0, np.float32)
    c, s, f, e = O.search_block(x, np.float32(0.1), -2, 6)
    assert s <= 126 and f <= 0


def test_tie_break_prefers_smaller_offset():
    """All-equal blocks where several scales represent the value exactly: every SSE is 0 and the
    smallest |f| (then the smallest f) must win."""
    for val in (3.0, 6.0, 1.5, 0.75):
        x = np.full(16, val, np.float32)
        g = np.float32(val / 6.0 / 1.0)  # makes the default scale exactly 1 * g... then d = 1 * g
        c, s, f, e = O.search_block(x, g, -2, 6)
        bf, bs, c0, tab = brute.search(x[None], g, -2, 6)
        assert f == bf[0] and e == bs[0]
    # exact ties with a nonzero error: dyadic blocks and a power-of-two tensor scale make many
    # candidates' SSEs coincide; per-offset windows [f, f] give each candidate's SSE.
    rng = np.random.default_rng(5)
    found = 0
    for trial in range(3000):
        x = (rng.integers(-24, 25, 16) / 8.0).astype(np.float32)
        if not np.any(x):
            continue
        g = np.float32(2.0 ** int(rng.integers(-8, -3)))
        per = []
        for f in range(-2, 7):
            c, s, ff, e = O.search_block(x, g, f, f)
            if ff != -128:
                per.append((np.float32(e), abs(f), f))
        per.sort()
        if len(per) > 1 and per[0][0] == per[1][0] and per[0][0] > 0:
            found += 1
            c, s, f, e = O.search_block(x, g, -2, 6)
            assert f == per[0][2] and np.float32(e) == per[0][0]
            bf, bs, c0, tab = brute.search(x[None], g, -2, 6)
            assert bf[0] == f
            if found >= 20:
                break
    assert found > 0


def test_dequantize_vs_library_decode():
    X = RNG.standard_normal(16 * 512).astype(np.float32)
    codes, scales, g, bf, bs = O.quantize(X, -2, 6)
    out = O.dequantize(codes, scales, g, O.F32)
    q = np.stack([codes & 0xF, codes >> 4], -1).reshape(-1).astype(np.uint8)
    v = q.view(md.float4_e2m1fn).astype(np.float32)
    d = (np.repeat(scales.view(md.float8_e4m3fn).astype(np.float32), 16) * g).astype(np.float32)
    ref = (v * d).astype(np.float32)
    assert np.array_equal(out.view(np.uint32), ref.view(np.uint32))
    # narrowed outputs are the RNE casts of the FP32 result
    assert np.array_equal(O.dequantize(codes, scales, g, O.BF16), ref.astype(md.bfloat16).view(np.uint16))
    assert np.array_equal(O.dequantize(codes, scales, g, O.F16), ref.astype(np.float16).view(np.uint16))
    # the normalised absolute error (BEVFormer page, section 7 metric) is in the FP4 range
    nae = np.abs(out - X).mean() / np.abs(X).mean()
    assert 0.05 < nae < 0.2
    # the poison scale byte dequantizes to NaN
    assert np.all(np.isnan(O.dequantize(np.zeros(8, np.uint8), np.array([0x7F], np.uint8), g)))


def _sylvester(n):
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def test_hadamard16_matches_matrix_and_is_an_involution():
    H = _sylvester(16) / 4.0
    X = RNG.standard_normal((256, 16)).astype(np.float32)
    out = O.hadamard16(X.reshape(-1)).reshape(-1, 16)
    ref = X.astype(np.float64) @ H.T
    assert np.allclose(out, ref, rtol=0, atol=8 * np.finfo(np.float32).eps * np.abs(X).sum(1, keepdims=True))
    # dyadic integers: every butterfly is exact, so the result equals the exact product
    Xi = RNG.integers(-64, 65, (256, 16)).astype(np.float32)
    outi = O.hadamard16(Xi.reshape(-1)).reshape(-1, 16)
    assert np.array_equal(outi, (Xi.astype(np.float64) @ H.T).astype(np.float32))
    # applying it twice returns the input exactly (H/4 is orthogonal and symmetric) on dyadic inputs
    assert np.array_equal(O.hadamard16(outi.reshape(-1)).reshape(-1, 16), Xi)
    # narrowed output: RNE of the FP32 result
    assert np.array_equal(O.hadamard16(X.reshape(-1), out_dtype=O.BF16), out.reshape(-1).astype(md.bfloat16).view(np.uint16))
    # bf16 input is widened exactly
    xb = X.reshape(-1).astype(md.bfloat16)
    assert np.array_equal(O.hadamard16(xb.view(np.uint16), dtype=O.BF16), O.hadamard16(xb.astype(np.float32)))


def test_hadamard16_sign_diagonal():
    """QuIP#-style H D: the forward map is (H/4) D, the inverse its transpose D (H/4)."""
    H = _sylvester(16) / 4.0
    Xi = RNG.integers(-64, 65, (256, 16)).astype(np.float32)
    for signs in (0x0001, 0x8000, 0xA5C3, 0xFFFF, int(RNG.integers(0, 1 << 16))):
        D = np.diag([-1.0 if (signs >> i) & 1 else 1.0 for i in range(16)])
        fwd = O.hadamard16_ex(Xi.reshape(-1), signs).reshape(-1, 16)
        assert np.array_equal(fwd, (Xi.astype(np.float64) @ (H @ D).T).astype(np.float32))
        inv = O.hadamard16_ex(Xi.reshape(-1), signs, inverse=True).reshape(-1, 16)
        assert np.array_equal(inv, (Xi.astype(np.float64) @ (D @ H).T).astype(np.float32))
        # the inverse undoes the forward map, and dot products of rotated pairs are unchanged
        assert np.array_equal(O.hadamard16_ex(fwd.reshape(-1), signs, inverse=True).reshape(-1, 16), Xi)
        assert np.array_equal((fwd[:128].astype(np.float64) * fwd[128:]).sum(1),
                              (Xi[:128].astype(np.float64) * Xi[128:]).sum(1))
    assert np.array_equal(O.hadamard16_ex(Xi.reshape(-1), 0), O.hadamard16(Xi.reshape(-1)))
    assert np.array_equal(O.hadamard16_ex(Xi.reshape(-1), 0, inverse=True), O.hadamard16(Xi.reshape(-1)))
    with pytest.raises(ValueError):
        O.hadamard16_ex(Xi.reshape(-1), 1 << 16)


def test_kv_mixed_layout():
    rng = np.random.default_rng(3)
    B, H, T, D = 1, 2, 80, 128
    k = rng.standard_normal((B, H, T, D)).astype(np.float32).astype(md.bfloat16)
    kb = k.view(np.uint16)
    so, ro, codes, scales, g = O.kv_mixed(kb, 16, 16, 1, -2, 6)
    assert np.array_equal(so, kb[:, :, :16])
    assert np.array_equal(ro, kb[:, :, -16:])
    mid = k[:, :, 16:-16].astype(np.float32)
    rot = O.hadamard16(np.ascontiguousarray(mid).reshape(-1)).reshape(mid.shape)
    assert g == np.float32(np.abs(rot).max() / np.float32(2688))
    c2, s2, g2, _, _ = O.quantize(rot.reshape(-1), -2, 6)
    assert np.array_equal(codes.reshape(-1), c2) and np.array_equal(scales.reshape(-1), s2)
    # without rotation the middle is the plain quantize of the BF16 values
    so, ro, codes, scales, g = O.kv_mixed(kb, 16, 16, 0, -2, 6)
    c3, s3, g3, _, _ = O.quantize(np.ascontiguousarray(mid).reshape(-1), -2, 6)
    assert g == g3 and np.array_equal(codes.reshape(-1), c3)


def test_tensor_amax_and_global_scale():
    x = RNG.standard_normal(10001).astype(np.float32)
    assert O.tensor_amax(x) == np.abs(x).max()
    assert O.global_scale(np.float32(2688.0)) == 1.0
    a = np.float32(3.7)
    assert O.global_scale(a) == np.float32(a / np.float32(2688.0))
    y = x.copy()
    y[17] = np.nan
    assert np.isnan(O.tensor_amax(y))
    y[17] = -np.inf
    assert np.isinf(O.tensor_amax(y))
    assert O.tensor_amax(np.zeros(0, np.float32)) == 0.0
    h = x.astype(np.float16)
    assert O.tensor_amax(h.view(np.uint16), O.F16) == np.abs(h).max().astype(np.float32)


def test_fullsize_harness_counts_planted_mismatches(tmp_path):
    """The whole-tensor comparison harness (spawned oracle workers over memory-mapped files) reports 0
    mismatches when the "device" outputs are the oracle's own, and exactly the planted ones otherwise."""
    from tests import fullsize as FS
    rng = np.random.default_rng(5)
    n = 16 * 3000
    x = (rng.standard_normal(n) * 2).astype(np.float32)
    xpath = str(tmp_path / "x.bin")
    x.tofile(xpath)
    g = O.global_scale(O.tensor_amax(x))
    rc, rs, rf, rse = O.quantize_blocks(x, 0, n // 16, g, -2, 6)
    rd = O.dequantize(rc, rs, g)
    paths = {}
    for k, a in (("codes", rc), ("scales", rs), ("f", rf), ("sse", rse), ("deq", rd)):
        paths[k] = str(tmp_path / (k + ".bin"))
        a.tofile(paths[k])
    tot = FS.oracle_compare(xpath, 0, n, g, -2, 6, paths, processes=3)
    assert tot["blocks"] == n // 16 and all(tot[k] == 0 for k in ("codes", "scales", "f", "sse", "deq"))
    assert np.array_equal(tot["hist"], np.bincount(rf.astype(np.int64) + 128, minlength=256))
    bad_c, bad_d = rc.copy(), rd.copy()
    bad_c[8 * 1234 + 3] ^= 0x10
    bad_d[16 * 2500 + 7] = np.nextafter(bad_d[16 * 2500 + 7], np.float32(np.inf))
    bad_c.tofile(paths["codes"])
    bad_d.tofile(paths["deq"])
    tot = FS.oracle_compare(xpath, 0, n, g, -2, 6, paths, processes=3)
    assert (tot["codes"], tot["codes_first"], tot["deq"], tot["deq_first"], tot["scales"]) == (1, 1234, 1, 2500, 0)


def test_certificate_blocks_are_adversarial_and_never_certified_wrongly():
    """tests/golden/certificate_blocks.txt: every "flip" block has its two best candidates ordered one way
    by the definition (oracle) and the other way by the kernel's fast score (exact emulation), every "tie"
    block has two best candidates with equal definition scores that the fast score tells apart, and the
    emulated certificate defers all of them; "edge" blocks, when certified, get the definition's winner.
    At least a few hundred such blocks (the GPU runs them in test_gpu_certificate_blocks)."""
    from tests import certblocks, fastscore as FSC
    rows = certblocks.load()
    kinds = {k: sum(1 for r in rows if r[0] == k) for k in ("flip", "tie", "edge")}
    assert kinds["flip"] >= 200 and kinds["tie"] >= 50 and kinds["edge"] >= 40, kinds
    for kind, g, f_lo, nc, x in rows:
        P = FSC.scores(x, g, f_lo, nc)
        F = {}
        for f in P:
            _, _, fs, sse = O.search_block(x, g, f, f)
            if fs == f:
                F[f] = float(sse)
        st, fc = FSC.certificate(x, g, f_lo, nc)
        win = min(F, key=lambda f: (F[f], abs(f), f)) if F else None
        if kind in ("flip", "tie"):
            a, b = sorted(F, key=lambda f: (F[f], abs(f), f))[:2]
            if kind == "flip":
                assert F[a] < F[b] and P[a] > P[b], (x, g)
            else:
                assert F[a] == F[b] and P[a] != P[b], (x, g)
            assert st == "deferred", (kind, x, g)
        elif st == "certified":
            assert fc == win, (x, g)
        assert O.search_block(x, g, f_lo, f_lo + nc - 1)[2] == (win if win is not None else -128)
