"""The step kernel's page selection is exact by construction: tensor-core
scores u with a rigorous half-width e (|u - U| <= e, U the oracle's
channel-order score) narrow the candidates, the survivors are rescored
exactly, and the cluster merges exact lists (QUEST page selection for the
active rows, LoSA paper, methodology; QUEST paper, query-aware page
selection).  This test runs that algorithm as a plain-Python model on the
CPU -- per CTA a contiguous page range, score chunks with a list carried
between them, group maxima of lower keys, the k-round lower bound of the
k-th largest, survivors by u + emax, the exact path on overflow, rescoring,
top k by rank, then the merge over the CTAs' lists -- and checks that it
returns exactly the oracle's top-k pages (value descending, lower page
first) on random, tied and adversarial scores.  A planted mistake (a strict
survivor test) must make it fail.  The GPU parity tests check the kernel."""
import numpy as np
import pytest

import oracle

U32 = 0xFFFFFFFF


def _rd_sub(a, b):
    """float32 a - b rounded toward -inf."""
    x = float(a) - float(b)
    f = np.float32(x)
    return np.nextafter(f, np.float32(-np.inf)) if float(f) > x else f


def _ru_add(a, b):
    """float32 a + b rounded toward +inf."""
    x = float(a) + float(b)
    f = np.float32(x)
    return np.nextafter(f, np.float32(np.inf)) if float(f) < x else f


def _obits(f):
    """Order-preserving uint32 of a float32 (-0 folded onto +0)."""
    b = int(np.float32(f).view(np.uint32))
    if b == 0x80000000:
        b = 0
    return (~b) & U32 if b & 0x80000000 else b | 0x80000000


def _ovalue(x):
    """The float32 whose ordered bits are x (x != 0)."""
    b = x & 0x7FFFFFFF if x & 0x80000000 else (~x) & U32
    return np.uint32(b).view(np.float32)


def _key(v, p):
    return (_obits(v) << 32) | ((~p) & U32)


def _kth_lb(gm, k):
    """The warp's k-round lower bound of the k-th largest of 64 group
    maxima held two per lane (0 = empty)."""
    gm = list(gm) + [0] * (64 - len(gm))
    h0 = [max(gm[l], gm[l + 32]) for l in range(32)]
    h1 = [min(gm[l], gm[l + 32]) for l in range(32)]
    m = 0
    for _ in range(k):
        m = max(h0)
        for l in range(32):
            if h0[l] == m:
                h0[l], h1[l] = h1[l], 0
    return m


def _cta_list(U, u, e, pages, k, spc, lb, strict=False):
    """One CTA's exact list (top min(k, n) keys) and threshold over `pages`
    (ascending global page ids), scored in chunks of spc pages."""
    lst, thr = [], 0
    gm = [0] * 64  # group maxima of lower-key value words, over all pages so far
    emax = np.float32(0)
    for c0 in range(0, len(pages), spc):
        chunk = pages[c0:c0 + spc]
        for j, p in enumerate(chunk):  # the scan: groups by position, half-widths
            g = (c0 + j) % 64
            gm[g] = max(gm[g], _obits(_rd_sub(u[p], e[p])))
            emax = max(emax, e[p])
        t = max(_kth_lb(gm, k), thr >> 32)
        tf = _ovalue(t) if t else np.float32(-np.inf)
        if strict:
            surv = [p for p in chunk if _ru_add(u[p], emax) > tf]
        else:
            surv = [p for p in chunk if _ru_add(u[p], emax) >= tf]
        if len(lst) + len(surv) > lb:  # the exact path: the chunk's exact top k
            keys = sorted((_key(U[p], p) for p in chunk), reverse=True)[:k]
        else:
            keys = [_key(U[p], p) for p in surv]  # rescored exactly
        cand = lst + keys
        ranked = sorted(cand, reverse=True)
        lst = ranked[:k]
        if len(ranked) >= k:
            thr = max(ranked[k - 1], thr)
    return lst, thr


def _select(U, u, e, k, C, spc, lb, strict=False):
    P = len(U)
    cp = ((P + C - 1) // C + 7) // 8 * 8
    lists = [_cta_list(U, u, e, list(range(c * cp, min(P, (c + 1) * cp))), k, spc, lb, strict)
             for c in range(C) if c * cp < P]
    tau = max(t for _, t in lists)
    keys = sorted((x for lst, _ in lists for x in lst if x >= tau), reverse=True)[:k]
    return sorted(((~x) & U32) for x in keys)


def _approx(rng, U, rel):
    """Tensor-core stand-ins: u within e of U (e > 0 per page)."""
    scale = np.abs(U).astype(np.float64).max() + 1.0
    e = (rel * scale * (0.5 + rng.random(len(U)))).astype(np.float32)
    d = (rng.random(len(U)) * 2 - 1) * 0.9 * e.astype(np.float64)
    u = (U.astype(np.float64) + d).astype(np.float32)
    bad = np.abs(u.astype(np.float64) - U.astype(np.float64)) > e.astype(np.float64)
    u[bad] = U[bad]
    return u, e


CASES = [
    # (P, k, C, spc, lb, kind, rel)
    (700, 8, 8, 64, 80, "normal", 1e-4),
    (4096, 8, 8, 512, 80, "normal", 6e-5),
    (1500, 16, 3, 128, 80, "normal", 1e-3),
    (257, 1, 5, 64, 72, "normal", 1e-2),
    (2000, 64, 8, 256, 128, "normal", 1e-4),
    (900, 8, 8, 64, 80, "ties", 1e-3),
    (3000, 16, 8, 512, 80, "ties", 1e-4),
    (600, 8, 2, 128, 80, "wide", 2.0),
    (1200, 8, 8, 128, 80, "adversarial", 1e-3),
]


def _scores(rng, P, kind):
    if kind == "ties":
        return rng.integers(-6, 7, size=P).astype(np.float32)
    if kind == "adversarial":
        U = rng.standard_normal(P).astype(np.float32)
        U[rng.integers(0, P, size=P // 4)] = np.float32(1.5)  # a large tied block
        U[rng.integers(0, P, size=8)] = np.float32(-0.0)
        return U
    return (rng.standard_normal(P) * 20).astype(np.float32)


@pytest.mark.parametrize("case", range(len(CASES)))
def test_model_selects_the_oracle_top_k(case):
    P, k, C, spc, lb, kind, rel = CASES[case]
    rng = np.random.default_rng(1000 + case)
    for _ in range(3):
        U = _scores(rng, P, kind)
        u, e = _approx(rng, U, rel)
        got = _select(U, u, e, k, C, spc, lb)
        want = sorted(oracle.topk_pages(U, k).tolist())
        assert got == want, (case, kind)


def test_planted_strict_survivor_test_is_caught():
    # distinct exact scores (intervals of width zero), one page per group:
    # the bound is then exactly the 8th largest score, and a strict survivor
    # test drops that page; the selection above must notice
    rng = np.random.default_rng(7)
    P, k = 64, 8
    U = rng.permutation(np.arange(P, dtype=np.float32) - 20.0)
    e = np.zeros(P, np.float32)
    want = sorted(oracle.topk_pages(U, k).tolist())
    assert _select(U, U.copy(), e, k, 1, 64, 80) == want
    assert _select(U, U.copy(), e, k, 1, 64, 80, strict=True) != want
