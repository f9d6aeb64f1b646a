"""Emulation, in exact binary32 arithmetic, of the search kernel's scaled-domain fast score and of the
certificate that decides whether the fast score alone may pick a block's scale (thread-per-block kernel,
windows of 9 or 17 offsets).  Used by the tests to build and check adversarial blocks: blocks where the
fast score P and the definition's score F order two candidates differently must never be certified.

Not the oracle: F always comes from the oracle; this module only mirrors the kernel's shortcut.  Every
operation is one correctly rounded binary32 operation (tests/exact_f32.py); the E2M1 and E4M3 roundings
are the ml_dtypes casts (round to nearest even, saturating)."""
from __future__ import annotations

from fractions import Fraction

import ml_dtypes
import numpy as np

from . import exact_f32 as X

INF = Fraction(10) ** 400


def _f32(q: Fraction) -> np.float32:
    return np.float32(float(q))


def e4m3_value(c: int) -> Fraction:
    return Fraction(float(np.array([c], np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)[0]))


def e2m1_value(y: Fraction) -> Fraction:
    return Fraction(float(np.array([float(y)], np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float32)[0]))


def c0_of(amax_b: Fraction, g: Fraction) -> int:
    """Default code E4M3(fl(fl(amax_b / 6) / g)), saturating at 448."""
    v = X.rne(X.rne(amax_b / 6) / g)
    v = min(v, Fraction(448))
    return int(np.array([float(v)], np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0])


def entry(c: int, g: Fraction):
    """The kernel's candidate-table entry of code c: (r, dd, d); r = 0 and dd = inf for unusable codes."""
    d = X.mul(e4m3_value(c), g) if 0 <= c <= 126 else Fraction(0)   # code 127 is NaN: never usable
    usable = 1 <= c <= 126 and d != 0
    r = X.rne(1 / d) if usable else Fraction(0)
    if usable and abs(r) > X.MAX:
        usable, r = False, Fraction(0)
    return (r, X.mul(d, d) if usable else INF, d)


def fast_score(x: list[Fraction], r: Fraction, dd: Fraction):
    """P = fl(fl(lo + hi) * dd): lo / hi are FMA chains over the even / odd elements of (v - y)^2 with
    y = fl(x r), v = E2M1(y) and v - y rounded once.  None for an unusable candidate (the kernel's NaN)."""
    if dd == INF:
        return None
    acc = [None, None]
    for i, xi in enumerate(x):
        y = X.mul(xi, r)
        e = X.rne(e2m1_value(y) - y)
        acc[i & 1] = X.mul(e, e) if acc[i & 1] is None else X.fma(e, e, acc[i & 1])
    return X.mul(X.add(acc[0], acc[1]), dd)


def _bits(q: Fraction) -> int:
    return int(np.array([float(q)], np.float32).view(np.uint32)[0])


def certificate(x16, g, f_lo: int, nc: int):
    """What the kernel's fast path does with this block: returns ("certified", f*) when the fast score
    alone decides (f* its choice), or ("deferred", reason) when the block goes to the definition."""
    x = [X.f(v) for v in np.asarray(x16, np.float32)]
    g = X.f(np.float32(g))
    amax_b = max(abs(v) for v in x)
    if amax_b == 0:
        return ("zero", None)
    c0 = c0_of(amax_b, g)
    clo, chi = c0 + f_lo, c0 + f_lo + nc - 1
    lo_ok = Fraction(2) ** -40 <= amax_b <= Fraction(2) ** 40
    if nc >= 17:
        if clo < -16 or chi > 127 + 16 or not lo_ok:
            return ("deferred", "range")
        vlo, vhi = max(clo, 1), min(chi, 126)
        if vlo > vhi:
            return ("deferred", "range")
    else:
        if clo < 1 or chi > 126 or not lo_ok:
            return ("deferred", "range")
        vlo, vhi = clo, chi
    r_lo, _, d_lo = entry(vlo, g)
    if r_lo == 0 or not d_lo >= Fraction(2) ** -40 or not X.mul(amax_b, r_lo) <= 1024:
        return ("deferred", "range")
    d_hi = entry(vhi, g)[2]
    keys = []
    for j in range(nc):
        r, dd, _ = entry(clo + j, g)
        s = fast_score(x, r, dd)
        if s is not None:
            keys.append(((_bits(s) & ~31) | j, j))
    keys.sort()
    if not keys or keys[0][0] >= 0x7F800000:
        return ("deferred", "no finite score")
    m1 = keys[0][0]
    pbest = Fraction(float(np.array([m1 & ~31], np.uint32).view(np.float32)[0]))
    if len(keys) > 1 and keys[1][0] < 0x7F800000:
        p2 = Fraction(float(np.array([keys[1][0] & ~31], np.uint32).view(np.float32)[0]))
    else:
        p2 = INF
    dmax = max(d_hi, X.fma(amax_b, X.f(np.float32(1.000001)), X.mul(Fraction(-6), d_lo)))
    beta = X.fma(amax_b, X.fma(amax_b, Fraction(2) ** -36, X.mul(dmax, Fraction(2) ** -15)), Fraction(2) ** -140)
    thr = X.fma(pbest, 1 + Fraction(2) ** -12, X.mul(beta, X.f(np.float32(2.51))))
    if not p2 > thr:
        return ("deferred", "near tie")
    return ("certified", f_lo + (m1 & 31))


def scores(x16, g, f_lo: int, nc: int):
    """{f: P_f} for the usable candidates of the window (exact binary32 emulation)."""
    x = [X.f(v) for v in np.asarray(x16, np.float32)]
    g = X.f(np.float32(g))
    c0 = c0_of(max(abs(v) for v in x), g)
    out = {}
    for j in range(nc):
        r, dd, _ = entry(c0 + f_lo + j, g)
        s = fast_score(x, r, dd)
        if s is not None:
            out[f_lo + j] = s
    return out
