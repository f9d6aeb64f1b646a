"""Writes tests/golden/certificate_blocks.txt: adversarial blocks for the search kernel's certified fast
score ("Search your block floating-point scales!", Method > ScaleSearch: the scale minimising the block
error wins; the kernel scores candidates in a scaled domain and may only skip the definition when that
score's order is certain).

Each block is built so that the definition's score F (the oracle) and the kernel's fast score P (the exact
emulation in tests/fastscore.py) order its two best candidates differently, or tie in F while P orders
them, or sits at an edge of the magnitude range the certificate covers.  F comes only from the oracle; P
only from the emulator.  Run from the repository root:

    python -m tests.golden.make_certificate_blocks
"""
from __future__ import annotations

import os

import ml_dtypes
import numpy as np

from oracle import oracle as O
from tests import fastscore as FSC

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "certificate_blocks.txt")
GS = [np.float32(4.7 / 2688), np.float32(2.0 ** -8), np.float32(3 * 2.0 ** -10), np.float32(0.0123)]
E4M3 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)


def e2m1(y):
    return y.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)


def c0s(x, g):
    a = np.abs(x).max(1)
    v = np.minimum((a / np.float32(6)) / g, np.float32(448)).astype(np.float32)
    return v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8).astype(np.int64)


def f_and_p(x, g, f_lo, nc):
    """numpy float32 evaluation of F (exact: IEEE binary32 per operation, in element order) and of an
    approximation of P (the FMA chain done in float64 then rounded), for every candidate; inf = unusable."""
    nb = x.shape[0]
    c0 = c0s(x, g)
    F = np.full((nb, nc), np.inf)
    P = np.full((nb, nc), np.inf)
    for j in range(nc):
        c = c0 + f_lo + j
        ok = (c >= 1) & (c <= 126)
        d = (E4M3[np.clip(c, 0, 127)] * g).astype(np.float32)
        with np.errstate(divide="ignore", over="ignore", invalid="ignore"):
            r = (np.float32(1) / d).astype(np.float32)
            y = (x * r[:, None]).astype(np.float32)
            v = e2m1(y)
            e = (x - (v * d[:, None]).astype(np.float32)).astype(np.float32)
            s = np.zeros(nb, np.float32)
            for i in range(16):
                s = (s + (e[:, i] * e[:, i]).astype(np.float32)).astype(np.float32)
            ev = (v - y).astype(np.float32).astype(np.float64)
            lo = np.zeros(nb)
            hi = np.zeros(nb)
            for i in range(0, 16, 2):
                lo = (lo + ev[:, i] ** 2).astype(np.float32).astype(np.float64)
                hi = (hi + ev[:, i + 1] ** 2).astype(np.float32).astype(np.float64)
            p = ((lo + hi).astype(np.float32) * (d * d).astype(np.float32)).astype(np.float32)
        ok &= np.isfinite(r) & (d != 0)
        F[:, j] = np.where(ok, s, np.inf)
        P[:, j] = np.where(ok, p, np.inf)
    return F, P


def exact_scores(x16, g, f_lo, nc):
    """F from the oracle (one-candidate windows) and P from the exact emulator, for every usable offset."""
    P = FSC.scores(x16, g, f_lo, nc)
    F = {}
    for f in P:
        _, _, fs, sse = O.search_block(x16, g, f, f)
        if fs == f:
            F[f] = float(sse)
    return F, {f: float(v) for f, v in P.items()}


def definition_winner(F):
    return min(F, key=lambda f: (F[f], abs(f), f))


def p_winner(P):
    return min(P, key=lambda f: (P[f], f - min(P)))   # P's key order: score, then window position


def find_flips(rng, g, f_lo, nc, want, dist):
    found = []
    tries = 0
    while len(found) < want and tries < 40:
        tries += 1
        if dist == "normal":
            x = rng.standard_normal((4096, 16)).astype(np.float32)
        elif dist == "t3":
            x = (rng.standard_normal((4096, 16)) / np.sqrt((rng.standard_normal((4096, 16, 3)) ** 2).mean(-1))).astype(np.float32)
        else:
            x = rng.uniform(-1, 1, (4096, 16)).astype(np.float32)
        x *= np.float32(g * 600)
        F, _ = f_and_p(x, g, f_lo, nc)
        order = np.argsort(F, 1)
        a, b = order[:, 0], order[:, 1]
        ok = np.isfinite(F[np.arange(len(x)), b])
        for i in np.flatnonzero(ok)[:400]:
            # move one element so that the two best candidates' F meet (quadratic model, codes fixed)
            xi = x[i].astype(np.float64)
            c0 = c0s(x[i:i + 1], g)[0]
            da = float(E4M3[c0 + f_lo + a[i]]) * float(g)
            db = float(E4M3[c0 + f_lo + b[i]]) * float(g)
            ea = xi - e2m1((x[i] / np.float32(da)).astype(np.float32)) * da
            eb = xi - e2m1((x[i] / np.float32(db)).astype(np.float32)) * db
            gap = F[i, a[i]] - F[i, b[i]]
            j = int(np.argmax(np.abs(ea - eb)))
            if abs(ea[j] - eb[j]) < 1e-30:
                continue
            t = np.float32(xi[j] - gap / (2 * (ea[j] - eb[j])))
            if not np.isfinite(t) or np.sign(t) != np.sign(x[i, j]) or abs(t) > np.abs(x[i]).max():
                continue
            cand = np.repeat(x[i:i + 1], 129, 0)
            ulps = np.arange(-64, 65)
            cand[:, j] = (t.view(np.int32) + ulps).astype(np.int32).view(np.float32)
            Fc, Pc = f_and_p(cand, g, f_lo, nc)
            for k in range(len(cand)):
                fa, fb, pa, pb = Fc[k, a[i]], Fc[k, b[i]], Pc[k, a[i]], Pc[k, b[i]]
                if (fa < fb) != (pa < pb) or fa == fb:
                    found.append(cand[k].copy())
            if len(found) >= want:
                break
    return found


def confirm(blocks, g, f_lo, nc):
    """Keep the blocks whose two best F candidates are ordered differently by P (or tie in F while P
    orders them), checked exactly; every kept block must be deferred by the certificate."""
    kept = []
    for x16 in blocks:
        F, P = exact_scores(x16, g, f_lo, nc)
        if len(F) < 2:
            continue
        w = definition_winner(F)
        best2 = sorted(F, key=lambda f: (F[f], abs(f), f))[:2]
        flip = (P[best2[0]] > P[best2[1]]) or (F[best2[0]] == F[best2[1]] and P[best2[0]] != P[best2[1]])
        if not flip:
            continue
        st, f = FSC.certificate(x16, g, f_lo, nc)
        if st == "certified":
            raise SystemExit(f"certificate accepted an order-flipping block (g={g!r}): {x16.tolist()}")
        kind = "tie" if F[best2[0]] == F[best2[1]] else "flip"
        kept.append((kind, x16, w))
    return kept


def edge_blocks(rng):
    """Blocks at the edges of the range the certificate covers: amax_b at 2^-40 and 2^40 (times 1 +- a
    few ulps), candidates with d near 2^-40, and small default codes whose window reaches the smallest
    scales (both window widths)."""
    out = []
    for amax in (2.0 ** -40, 2.0 ** 40):
        for k in (-2, -1, 0, 1, 2):
            base = rng.standard_normal(16).astype(np.float32)
            base /= np.abs(base).max()
            a = np.float32(amax)
            a = (a.view(np.int32) + k).astype(np.int32).view(np.float32)
            x = (base * a).astype(np.float32)
            x[np.argmax(np.abs(x))] = a * np.sign(x[np.argmax(np.abs(x))])
            for g in (np.float32(float(a) / 6 / 100), np.float32(float(a) / 6 / 3)):
                for f_lo, nc in ((-2, 9), (-8, 17)):
                    out.append(("edge", x, g, f_lo, nc))
    for c0 in (1, 2, 3, 5, 9, 12):
        for f_lo, nc in ((-2, 9), (-8, 17)):
            g = np.float32(2.0 ** -8)
            a = np.float32(float(E4M3[c0]) * 6 * float(g))
            x = (rng.standard_normal(16) * float(a) / 3).astype(np.float32)
            x[0] = a
            out.append(("edge", x, g, f_lo, nc))
    return out


def hexf(v) -> str:
    """Shortest hex spelling of a binary32 value (trailing zero digits dropped)."""
    h = float(v).hex()
    if "p" in h and "." in h:
        m, e = h.split("p")
        h = m.rstrip("0").rstrip(".") + "p" + e
    return h


def main():
    rng = np.random.default_rng(2024)
    rows = []
    for g in GS:
        for f_lo, nc, dist in ((-2, 9, "normal"), (-2, 9, "t3"), (-2, 9, "uniform"), (-8, 17, "normal")):
            blocks = find_flips(rng, g, f_lo, nc, 40, dist)
            for kind, x16, w in confirm(blocks, g, f_lo, nc):
                rows.append((kind, x16, g, f_lo, nc))
    for kind, x16, g, f_lo, nc in edge_blocks(rng):
        st, _ = FSC.certificate(x16, g, f_lo, nc)
        F, P = exact_scores(x16, g, f_lo, nc) if st != "zero" else ({}, {})
        if st == "certified" and F and P and definition_winner(F) != p_winner(P):
            raise SystemExit(f"certificate accepted an edge block it gets wrong: {x16.tolist()}")
        rows.append((kind, x16, g, f_lo, nc))
    with open(OUT, "w") as fh:
        fh.write("# Adversarial blocks for the search kernel's certified fast score (written by\n"
                 "# tests/golden/make_certificate_blocks.py from the oracle and tests/fastscore.py only).\n"
                 "# \"Search your block floating-point scales!\", Method > ScaleSearch.  kind: flip = the fast score\n"
                 "# orders the two best candidates against the definition; tie = equal definition scores that the\n"
                 "# fast score orders; edge = a block at the edge of the magnitude range the certificate covers.\n"
                 "# columns: kind g f_lo n_offsets x0 .. x15 (binary32 as hex)\n")
        for kind, x16, g, f_lo, nc in rows:
            fh.write(" ".join([kind, hexf(g), str(f_lo), str(nc)] + [hexf(v) for v in x16]) + "\n")
    kinds = {k: sum(1 for r in rows if r[0] == k) for k in ("flip", "tie", "edge")}
    print(f"wrote {len(rows)} blocks to {OUT}: {kinds}")


if __name__ == "__main__":
    main()
