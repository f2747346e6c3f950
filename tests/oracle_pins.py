"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` function raises AssertionError when the oracle disagrees with
a hand-derived value (``tests/golden``), a closed form, an invariant, or a
brute-force numpy computation written independently of the oracle's C code.
``test_oracle_pins.py`` runs them; ``test_oracle_mutations.py`` plants bugs in
the oracle and checks that at least one pin catches each.
"""
from __future__ import annotations

import json
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# independent numpy brute force (fp64)
# ---------------------------------------------------------------------------
def np_attend(q, K, V, scale):
    s = scale * (K.astype(np.float64) @ q.astype(np.float64))
    m = s.max()
    w = np.exp(s - m)
    return (w @ V.astype(np.float64)) / w.sum(), m + np.log(w.sum())


def np_bound(q, kmin, kmax):
    q = q.astype(np.float64)
    return np.maximum(q * kmax.astype(np.float64), q * kmin.astype(np.float64)).sum(-1)


def rand_shape(rng, S=2, Hq=4, Hkv=2, d=16, L=45, ps=4, B=6, A=2, budget=12, scale=None,
               flags=0):
    return oracle.shape(S, Hq, Hkv, d, L, ps, B, A, budget,
                        scale if scale is not None else float(np.float32(0.37)), flags)


def rand_inputs(rng, sh):
    f = lambda *s: rng.standard_normal(s).astype(np.float32)
    Qp = f(sh.S, sh.Hq, sh.B, sh.d)
    Qc = Qp + np.float32(0.01) * f(sh.S, sh.Hq, sh.B, sh.d)
    # give a few tokens per head a large change
    for s in range(sh.S):
        for h in range(sh.Hq):
            idx = rng.choice(sh.B, size=min(sh.A + 1, sh.B), replace=False)
            Qc[s, h, idx] += f(len(idx), sh.d)
    return {"Qc": Qc.astype(np.float32), "Qp": Qp, "K": f(sh.S, sh.Hkv, sh.L, sh.d),
            "V": f(sh.S, sh.Hkv, sh.L, sh.d), "Kb": f(sh.S, sh.Hkv, sh.B, sh.d),
            "Vb": f(sh.S, sh.Hkv, sh.B, sh.d)}


def close(a, b, tol, what):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3g} > {tol}"


# ---------------------------------------------------------------------------
# golden, hand-derived
# ---------------------------------------------------------------------------
def pin_golden_attention():
    g = golden("attention_two_keys.json")
    o, lse = oracle.attend_tokens(np.array(g["q"]), np.array(g["K"]), np.array(g["V"]),
                                  [0, 1], g["scale"])
    close(o, g["expect_o"], 1e-7, "golden attention o")
    close(lse, g["expect_lse"], 1e-7, "golden attention lse")


def pin_golden_merge():
    g = golden("merge_two_parts.json")
    o, lse = oracle.merge(g["o1"], g["l1"], g["o2"], g["l2"])
    close(o, g["expect_o"], 1e-12, "golden merge o")
    close(lse, g["expect_lse"], 1e-12, "golden merge lse")


def pin_golden_bound():
    g = golden("quest_bound_pages.json")
    K = np.array(g["K"], np.float32)
    d = K.shape[1]
    sh = oracle.shape(1, 1, 1, d, K.shape[0], g["page_size"], 1, 1, 2)
    kmin, kmax = oracle.build_meta(sh, K[None, None])
    close(kmin[0, 0], g["expect_kmin"], 0, "golden kmin")
    close(kmax[0, 0], g["expect_kmax"], 0, "golden kmax")
    U = oracle.bound_scores(np.array(g["q"], np.float32), kmin[0, 0], kmax[0, 0])
    close(U, g["expect_U"], 0, "golden bound")
    for k, pages in g["expect_topk"].items():
        got = oracle.topk_pages(U, int(k))
        assert list(got) == pages, f"golden top-{k}: {list(got)} != {pages}"


def pin_golden_locality():
    g = golden("locality_active.json")
    Qc = np.array(g["Qc"], np.float32)[None, None]
    Qp = np.array(g["Qp"], np.float32)[None, None]
    B, d = Qc.shape[2], Qc.shape[3]
    sh = oracle.shape(1, 1, 1, d, 1, 1, B, 1, 1)
    mse = oracle.locality(sh, Qc, Qp)
    close(mse[0, 0], g["expect_mse"], 0, "golden mse")
    for a, toks in g["expect_active"].items():
        sh.A = int(a)
        got = oracle.active(sh, mse)
        assert list(got[0, 0]) == toks, f"golden active top-{a}: {list(got[0, 0])} != {toks}"


# ---------------------------------------------------------------------------
# brute force / closed forms / invariants
# ---------------------------------------------------------------------------
def pin_meta_bruteforce():
    rng = np.random.default_rng(11)
    sh = rand_shape(rng, L=45, ps=4)      # 12 pages, last one holds 1 token
    K = rng.standard_normal((sh.S, sh.Hkv, sh.L, sh.d)).astype(np.float32)
    kmin, kmax = oracle.build_meta(sh, K)
    P = oracle.n_pages(sh)
    for p in range(P):
        blk = K[:, :, p * sh.ps:min((p + 1) * sh.ps, sh.L), :]
        close(kmin[:, :, p], blk.min(axis=2), 0, f"kmin page {p}")
        close(kmax[:, :, p], blk.max(axis=2), 0, f"kmax page {p}")
        assert np.all(kmin[:, :, p, None] <= blk) and np.all(blk <= kmax[:, :, p, None])


def pin_attend_numpy():
    rng = np.random.default_rng(12)
    d, n = 24, 57
    q = rng.standard_normal(d).astype(np.float32)
    K = (3 * rng.standard_normal((n, d))).astype(np.float32)
    V = rng.standard_normal((n, d)).astype(np.float32)
    tok = rng.choice(n, size=31, replace=False)
    scale = 0.29
    o, lse = oracle.attend_tokens(q, K, V, tok, scale)
    ro, rl = np_attend(q, K[tok], V[tok], np.float64(np.float32(scale)))
    close(o, ro, 1e-12, "attend o vs numpy")
    close(lse, rl, 1e-12, "attend lse vs numpy")


def pin_merge_concat():
    """merge(attn(q,K1,V1), attn(q,K2,V2)) == attn(q, K1+K2, V1+V2)."""
    rng = np.random.default_rng(13)
    d = 32
    q = rng.standard_normal(d).astype(np.float32)
    K = (2 * rng.standard_normal((40, d))).astype(np.float32)
    V = rng.standard_normal((40, d)).astype(np.float32)
    scale = 0.5
    o1, l1 = oracle.attend_tokens(q, K, V, np.arange(0, 13), scale)
    o2, l2 = oracle.attend_tokens(q, K, V, np.arange(13, 40), scale)
    o, lse = oracle.merge(o1, l1, o2, l2)
    ro, rl = np_attend(q, K, V, scale)
    close(o, ro, 1e-12, "merge == attention over the union (o)")
    close(lse, rl, 1e-12, "merge == attention over the union (lse)")


def pin_bound_upper():
    """U(q,p) >= max_{j in p} q.k_j for every page."""
    rng = np.random.default_rng(14)
    d, ps, P = 64, 16, 40
    for trial in range(4):
        K = rng.standard_normal((P * ps, d)).astype(np.float32)
        q = rng.standard_normal(d).astype(np.float32)
        sh = oracle.shape(1, 1, 1, d, P * ps, ps, 1, 1, ps)
        kmin, kmax = oracle.build_meta(sh, K[None, None])
        U = oracle.bound_scores(q, kmin[0, 0], kmax[0, 0]).astype(np.float64)
        true = (K.astype(np.float64) @ q.astype(np.float64)).reshape(P, ps).max(1)
        tol = 1e-5 * (np.abs(q) @ np.maximum(np.abs(kmax[0, 0]), np.abs(kmin[0, 0])).T)
        assert np.all(U >= true - tol), f"bound below true max by {np.max(true - U):.3g}"
        close(U, np_bound(q, kmin[0, 0], kmax[0, 0]), float(np.max(tol)), "bound vs fp64")


def pin_bound_ps1_exact():
    """Page size 1: the bound is q.k itself; top-k pages = exact top-k tokens.
    Small integers keep every fp32 product and partial sum exact."""
    rng = np.random.default_rng(15)
    d, L = 32, 300
    K = rng.integers(-8, 9, size=(L, d)).astype(np.float32)
    q = rng.integers(-8, 9, size=d).astype(np.float32)
    sh = oracle.shape(1, 1, 1, d, L, 1, 1, 1, 1)
    kmin, kmax = oracle.build_meta(sh, K[None, None])
    U = oracle.bound_scores(q, kmin[0, 0], kmax[0, 0])
    exact = K.astype(np.int64) @ q.astype(np.int64)
    close(U, exact, 0, "ps=1 bound == q.k")
    for k in (1, 5, 17):
        order = np.lexsort((np.arange(L), -exact))  # score desc, index asc
        want = np.sort(order[:k])
        got = oracle.topk_pages(U, k)
        assert list(got) == list(want), f"ps=1 top-{k}: {got} != {want}"


def pin_locality_numpy():
    rng = np.random.default_rng(16)
    sh = rand_shape(rng, B=12, A=3, d=128)
    x = rand_inputs(rng, sh)
    mse = oracle.locality(sh, x["Qc"], x["Qp"])
    ref = ((x["Qc"].astype(np.float64) - x["Qp"].astype(np.float64)) ** 2).mean(-1)
    assert np.all(np.abs(mse - ref) <= 1e-5 * ref + 1e-12), "mse vs fp64"
    act = oracle.active(sh, mse)
    for s in range(sh.S):
        for h in range(sh.Hq):
            order = np.lexsort((np.arange(sh.B), -ref[s, h]))
            gaps = np.abs(np.diff(np.sort(ref[s, h])))
            if gaps.min() > 1e-4 * ref[s, h].max():
                assert list(act[s, h]) == sorted(order[:sh.A]), "active set vs fp64 ranking"


def pin_planted_recovery():
    """Planted actives (drift 1.0 vs 0.01) are recovered exactly on the tiny
    workload and on the first heads of the GQA workload."""
    from sparse_long_context_mse_b200 import synth
    for w in (synth.TINY, synth.GQA16K):
        cfg = synth.workload(w)
        if w == synth.GQA16K:
            cfg = cfg.with_(prefix_len=64)
        q = synth.gen_queries(cfg)
        sh = oracle.shape_of(cfg)
        mse = oracle.locality(sh, q["q"][1], q["q"][0])
        act = oracle.active(sh, mse)
        planted = q["planted"][0].numpy()
        for s in range(cfg.num_seqs):
            for h in range(cfg.n_q_heads):
                want = list(np.nonzero(planted[s, h])[0])
                assert list(act[s, h]) == want, f"{w} s{s} h{h}: {list(act[s, h])} != {want}"


def _np_dense_all(sh, x):
    """numpy: prefix attention per row, and attention over prefix + block."""
    G = sh.Hq // sh.Hkv
    o_p = np.zeros((sh.S, sh.Hq, sh.B, sh.d))
    l_p = np.zeros((sh.S, sh.Hq, sh.B))
    full = np.zeros_like(o_p)
    full_l = np.zeros_like(l_p)
    for s in range(sh.S):
        for h in range(sh.Hq):
            g = h // G
            Kc = np.concatenate([x["K"][s, g], x["Kb"][s, g]])
            Vc = np.concatenate([x["V"][s, g], x["Vb"][s, g]])
            for t in range(sh.B):
                q = x["Qc"][s, h, t]
                o_p[s, h, t], l_p[s, h, t] = np_attend(q, x["K"][s, g], x["V"][s, g], sh.scale)
                full[s, h, t], full_l[s, h, t] = np_attend(q, Kc, Vc, sh.scale)
    return o_p, l_p, full, full_l


def pin_dense_prefix_numpy():
    rng = np.random.default_rng(17)
    sh = rand_shape(rng)
    x = rand_inputs(rng, sh)
    r = oracle.dense_prefix(sh, x["Qc"], x["K"], x["V"], x["Kb"], x["Vb"])
    o_p, l_p, full, full_l = _np_dense_all(sh, x)
    close(r["o_p"], o_p, 1e-6, "dense o_p vs numpy")
    close(r["l_p"], l_p, 1e-6, "dense L_p vs numpy")
    close(r["out"], full, 1e-6, "dense out == attention over prefix+block")
    close(r["lse"], full_l, 1e-5, "dense lse == logsumexp over prefix+block")


def pin_dense_rows_numpy():
    """Row-by-row dense prefix attention (the checker of sampled stable rows
    at sizes where the full pass is too slow): rows from several sequences and
    heads of a GQA shape, in shuffled order, against numpy over each row's own
    KV head, and bitwise against the same rows of the full pass."""
    rng = np.random.default_rng(23)
    sh = rand_shape(rng, S=3, Hq=6, Hkv=2, L=37, B=5)
    x = rand_inputs(rng, sh)
    for g in range(sh.Hkv):  # very different KV heads: a wrong head shows at once
        x["V"][:, g] += np.float32(7.0 * (g + 1))
    for s in range(sh.S):
        x["V"][s] += np.float32(50.0 * s)
    n = sh.S * sh.Hq * sh.B
    rows = rng.permutation(n)[: n - 7].astype(np.int32)
    o_r, l_r = oracle.dense_rows(sh, x["Qc"], x["K"], x["V"], rows)
    G = sh.Hq // sh.Hkv
    for a, r in enumerate(rows):
        s, rem = divmod(int(r), sh.Hq * sh.B)
        h, t = divmod(rem, sh.B)
        o, L = np_attend(x["Qc"][s, h, t], x["K"][s, h // G], x["V"][s, h // G], sh.scale)
        close(o_r[a], o, 1e-6 * max(1.0, float(np.abs(o).max())), f"dense row {r} o_p vs numpy")
        close(l_r[a], L, 1e-5, f"dense row {r} L_p vs numpy")
    full = oracle.dense_prefix(sh, x["Qc"], x["K"], x["V"], x["Kb"], x["Vb"])
    fo = full["o_p"].reshape(n, sh.d)[rows]
    fl = full["l_p"].reshape(n)[rows]
    assert np.array_equal(o_r.view(np.uint32), fo.view(np.uint32)), "dense rows != full pass"
    assert np.array_equal(l_r.view(np.uint32), fl.view(np.uint32)), "dense rows L != full pass"


def pin_gqa_mapping():
    """Query head h reads KV head h // G: make the KV heads very different."""
    rng = np.random.default_rng(18)
    sh = rand_shape(rng, S=1, Hq=6, Hkv=3, L=20, B=3)
    x = rand_inputs(rng, sh)
    for g in range(sh.Hkv):
        x["V"][0, g] += np.float32(10.0 * (g + 1))
    r = oracle.dense_prefix(sh, x["Qc"], x["K"], x["V"], x["Kb"], x["Vb"])
    o_p, l_p, _, _ = _np_dense_all(sh, x)
    close(r["o_p"], o_p, 1e-5, "GQA mapping (o_p)")


def _step_inputs(seed, **kw):
    rng = np.random.default_rng(seed)
    sh = rand_shape(rng, **kw)
    x = rand_inputs(rng, sh)
    kmin, kmax = oracle.build_meta(sh, x["K"])
    cache = oracle.dense_prefix(sh, x["Qp"], x["K"], x["V"], x["Kb"], x["Vb"])
    return sh, x, kmin, kmax, cache


def pin_step_dense_equiv():
    """|A| = B and a budget covering the prefix: LoSA == dense attention."""
    sh, x, kmin, kmax, cache = _step_inputs(19, A=6, B=6, budget=10_000)
    r = oracle.step(sh, x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"],
                    cache["o_p"], cache["l_p"])
    o_p, l_p, full, full_l = _np_dense_all(sh, x)
    close(r["o_p"], o_p, 1e-6, "dense-equivalent step o_p")
    close(r["l_p"], l_p, 1e-5, "dense-equivalent step L_p")
    close(r["out"], full, 1e-6, "dense-equivalent step out")
    P = oracle.n_pages(sh)
    assert np.all(r["union_count"] == P)


def _np_suffix(sh, x, s, h, t):
    G = sh.Hq // sh.Hkv
    return np_attend(x["Qc"][s, h, t], x["Kb"][s, h // G], x["Vb"][s, h // G], sh.scale)


def _np_merge(o1, l1, o2, l2):
    m = max(l1, l2)
    a, b = np.exp(l1 - m), np.exp(l2 - m)
    return (a * o1 + b * o2) / (a + b), m + np.log(a + b)


def pin_step_stable_rows():
    """Stable rows: cache bitwise unchanged, out = merge(cached, fresh suffix)."""
    sh, x, kmin, kmax, cache = _step_inputs(20)
    r = oracle.step(sh, x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"],
                    cache["o_p"], cache["l_p"])
    n_stable = 0
    for s in range(sh.S):
        for h in range(sh.Hq):
            act = set(r["active_idx"][s, h].tolist())
            for t in range(sh.B):
                if t in act:
                    continue
                n_stable += 1
                assert np.array_equal(r["o_p"][s, h, t].view(np.uint32),
                                      cache["o_p"][s, h, t].view(np.uint32))
                assert r["l_p"][s, h, t].view(np.uint32) == cache["l_p"][s, h, t].view(np.uint32)
                os_, ls = _np_suffix(sh, x, s, h, t)
                o, l = _np_merge(cache["o_p"][s, h, t].astype(np.float64),
                                 float(cache["l_p"][s, h, t]), os_, ls)
                close(r["out"][s, h, t], o, 1e-6, "stable row out")
                close(r["lse"][s, h, t], l, 1e-5, "stable row lse")
    assert n_stable == sh.S * sh.Hq * (sh.B - sh.A)


def pin_step_zero_active():
    sh, x, kmin, kmax, cache = _step_inputs(21, A=0)
    r = oracle.step(sh, x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"],
                    cache["o_p"], cache["l_p"])
    assert np.array_equal(r["o_p"], cache["o_p"]) and np.array_equal(r["l_p"], cache["l_p"])
    for s in range(sh.S):
        for h in range(sh.Hq):
            for t in range(sh.B):
                os_, ls = _np_suffix(sh, x, s, h, t)
                o, _ = _np_merge(cache["o_p"][s, h, t].astype(np.float64),
                                 float(cache["l_p"][s, h, t]), os_, ls)
                close(r["out"][s, h, t], o, 1e-6, "|A|=0 row out")
    assert np.all(r["union_count"] == 0)


def pin_step_active_rows_bruteforce():
    """Active rows: pages are a top-k of the fp64 bound (ties within rounding
    allowed), o_p/L_p equal numpy attention over those pages' tokens, and the
    union count equals a brute-force set union with k <= U <= min(P, R k)."""
    sh, x, kmin, kmax, cache = _step_inputs(22, L=93, ps=4, B=8, A=3, budget=16)
    r = oracle.step(sh, x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"],
                    cache["o_p"], cache["l_p"])
    G = sh.Hq // sh.Hkv
    k = oracle.pages_per_row(sh)
    P = oracle.n_pages(sh)
    for s in range(sh.S):
        unions = [set() for _ in range(sh.Hkv)]
        for h in range(sh.Hq):
            g = h // G
            for a, t in enumerate(r["active_idx"][s, h]):
                q = x["Qc"][s, h, t]
                U = np_bound(q, kmin[s, g], kmax[s, g])
                pages = r["page_idx"][s, h, a]
                assert len(set(pages.tolist())) == k and list(pages) == sorted(pages)
                kth = np.sort(U)[::-1][k - 1]
                tol = 1e-5 * np.abs(U).max()
                assert np.all(U[pages] >= kth - tol), "selected page below the k-th bound"
                others = np.setdiff1d(np.arange(P), pages)
                assert np.all(U[others] <= kth + tol), "unselected page above the k-th bound"
                tok = np.concatenate([np.arange(p * sh.ps, min((p + 1) * sh.ps, sh.L))
                                      for p in pages])
                o, l = np_attend(q, x["K"][s, g][tok], x["V"][s, g][tok], sh.scale)
                close(r["o_p"][s, h, t], o, 1e-6, "active row o_p")
                close(r["l_p"][s, h, t], l, 1e-5, "active row L_p")
                os_, ls = _np_suffix(sh, x, s, h, t)
                om, _ = _np_merge(r["o_p"][s, h, t].astype(np.float64), float(r["l_p"][s, h, t]),
                                  os_, ls)
                close(r["out"][s, h, t], om, 1e-6, "active row out")
                unions[g].update(pages.tolist())
        for g in range(sh.Hkv):
            assert r["union_count"][s, g] == len(unions[g]), "union count vs set union"
            assert k <= r["union_count"][s, g] <= min(P, G * sh.A * k)


def pin_step_attend_union_bruteforce():
    """Variant: every active row attends to its group's whole page union.
    The selection is the default's; o_p/L_p equal numpy attention over the
    union's tokens (the union built here from page_idx); L_p is at least the
    default's (log-sum-exp over a superset of the row's own tokens)."""
    kw = dict(L=93, ps=4, B=8, A=3, budget=16)
    sh, x, kmin, kmax, cache = _step_inputs(23, **kw)
    shu, _, _, _, _ = _step_inputs(23, flags=oracle.ATTEND_UNION, **kw)
    args = (x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"], cache["o_p"],
            cache["l_p"])
    r0 = oracle.step(sh, *args)
    r = oracle.step(shu, *args)
    for key in ("active_idx", "page_idx", "union_count"):
        assert np.array_equal(r[key], r0[key]), key
    G = sh.Hq // sh.Hkv
    n_strict = 0
    for s in range(sh.S):
        for g in range(sh.Hkv):
            pages = sorted(set(r["page_idx"][s, g * G:(g + 1) * G].reshape(-1).tolist()))
            tok = np.concatenate([np.arange(p * sh.ps, min((p + 1) * sh.ps, sh.L)) for p in pages])
            for h in range(g * G, (g + 1) * G):
                for t in r["active_idx"][s, h]:
                    o, l = np_attend(x["Qc"][s, h, t], x["K"][s, g][tok], x["V"][s, g][tok],
                                     sh.scale)
                    close(r["o_p"][s, h, t], o, 1e-6, "union row o_p")
                    close(r["l_p"][s, h, t], l, 1e-5, "union row L_p")
                    assert r["l_p"][s, h, t] >= r0["l_p"][s, h, t] - 1e-5
                    n_strict += r["l_p"][s, h, t] > r0["l_p"][s, h, t] + 1e-4
    assert n_strict > 0, "the union added no tokens anywhere: the case does not test the variant"


def pin_step_attend_union_single_row():
    """With one active row per group (G = 1, |A| = 1) the union is the row's
    own pages: the variant equals the default step."""
    kw = dict(Hq=2, Hkv=2, A=1, L=61, budget=12)
    sh, x, kmin, kmax, cache = _step_inputs(24, **kw)
    shu, _, _, _, _ = _step_inputs(24, flags=oracle.ATTEND_UNION, **kw)
    args = (x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"], cache["o_p"],
            cache["l_p"])
    r0, r = oracle.step(sh, *args), oracle.step(shu, *args)
    for key in ("o_p", "l_p", "out", "lse", "page_idx"):
        assert np.array_equal(r[key], r0[key]), key


def pin_refresh_ref_rows():
    """Drift-safe reference: exactly the active rows take the current query
    (bitwise); every other row keeps its reference."""
    sh, x, kmin, kmax, cache = _step_inputs(25)
    q_ref = x["Qp"] + np.float32(0.5)
    r = oracle.step_ref(sh, x["Qc"], q_ref, x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"],
                        cache["o_p"], cache["l_p"])
    for s in range(sh.S):
        for h in range(sh.Hq):
            act = set(r["active_idx"][s, h].tolist())
            for t in range(sh.B):
                want = x["Qc"][s, h, t] if t in act else q_ref[s, h, t]
                assert np.array_equal(r["q_ref"][s, h, t].view(np.uint32), want.view(np.uint32))


def pin_drift_safe_slow_drift():
    """A token drifting slowly in one direction: against the previous step it
    never changes most, so plain locality never activates it; against its
    reference (the query its cached state came from) the change grows as
    n*delta and it becomes active at the first step with n*delta > the jump
    size of the other tokens -- step 4 for delta = 0.3, jump = 1 (closed form
    below)."""
    d, B = 16, 4
    sh = oracle.shape(1, 1, 1, d, 32, 4, B, 1, 8, float(np.float32(0.25)))
    rng = np.random.default_rng(26)
    u = np.zeros(d, np.float32)
    u[0] = 1.0
    K = rng.standard_normal((1, 1, 32, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, 32, d)).astype(np.float32)
    Kb = rng.standard_normal((1, 1, B, d)).astype(np.float32)
    Vb = rng.standard_normal((1, 1, B, d)).astype(np.float32)
    kmin, kmax = oracle.build_meta(sh, K)
    q1 = rng.standard_normal((1, 1, B, d)).astype(np.float32)
    cache = oracle.dense_prefix(sh, q1, K, V, Kb, Vb)
    delta, jump = np.float32(0.3), np.float32(1.0)
    prev, ref = q1, q1.copy()
    o_p, l_p = cache["o_p"], cache["l_p"]
    o_p2, l_p2 = o_p, l_p
    first_plain, first_safe = None, None
    for n in range(1, 7):
        cur = prev.copy()
        cur[0, 0, 0] += delta * u                      # token 0: slow drift
        j = 1 + (n - 1) % (B - 1)                      # one other token jumps by `jump`
        e = np.zeros(d, np.float32)
        e[1 + n % (d - 1)] = jump
        cur[0, 0, j] += e
        rp = oracle.step(sh, cur, prev, K, V, kmin, kmax, Kb, Vb, o_p, l_p)
        rs = oracle.step_ref(sh, cur, ref, K, V, kmin, kmax, Kb, Vb, o_p2, l_p2)
        if first_plain is None and 0 in rp["active_idx"][0, 0].tolist():
            first_plain = n
        if first_safe is None and 0 in rs["active_idx"][0, 0].tolist():
            first_safe = n
        prev, ref = cur, rs["q_ref"]
        o_p, l_p, o_p2, l_p2 = rp["o_p"], rp["l_p"], rs["o_p"], rs["l_p"]
    # token 0's change against its reference after n steps is n*delta in one
    # channel; a jumping token changes by `jump`: first n with n*delta > jump
    want = int(np.floor(float(jump) / float(delta))) + 1
    assert first_plain is None, first_plain
    assert first_safe == want, (first_safe, want)


def pin_append_then_meta():
    """Prefix growth: the grown prefix holds the old tokens then the block's
    (bitwise); pages entirely below the old length keep their records; the
    rebuilt pages bound every token they hold (brute force)."""
    rng = np.random.default_rng(27)
    S, Hkv, d, L, ps, B = 2, 2, 16, 45, 4, 6
    f = lambda *s_: rng.standard_normal(s_).astype(np.float32)
    K, V, Kb, Vb = f(S, Hkv, L, d), f(S, Hkv, L, d), f(S, Hkv, B, d), f(S, Hkv, B, d)
    K2, V2 = oracle.append_block(K, V, Kb, Vb)
    assert K2.shape == (S, Hkv, L + B, d)
    assert np.array_equal(K2[:, :, :L].view(np.uint32), K.view(np.uint32))
    assert np.array_equal(K2[:, :, L:].view(np.uint32), Kb.view(np.uint32))
    assert np.array_equal(V2[:, :, L:].view(np.uint32), Vb.view(np.uint32))
    sh1 = oracle.shape(S, 2 * Hkv, Hkv, d, L, ps, B, 2, 8)
    sh2 = oracle.shape(S, 2 * Hkv, Hkv, d, L + B, ps, B, 2, 8)
    mn1, mx1 = oracle.build_meta(sh1, K)
    mn2, mx2 = oracle.build_meta(sh2, K2)
    full = L // ps  # pages entirely below L
    assert np.array_equal(mn2[:, :, :full], mn1[:, :, :full])
    assert np.array_equal(mx2[:, :, :full], mx1[:, :, :full])
    for p in range(full, oracle.n_pages(sh2)):
        tok = K2[:, :, p * ps:min((p + 1) * ps, L + B)]
        assert np.array_equal(mn2[:, :, p], tok.min(axis=2))
        assert np.array_equal(mx2[:, :, p], tok.max(axis=2))


def pin_varlen_equal_lengths():
    """A variable-length batch whose lengths all equal L is the batched call,
    bit for bit (metadata, dense pass and step)."""
    sh, x, kmin, kmax, cache = _step_inputs(31, S=3)
    lens = [sh.L] * sh.S
    for (mn, mx), s in zip(oracle.build_meta_varlen(sh, lens, x["K"]), range(sh.S)):
        assert np.array_equal(mn, kmin[s:s + 1]) and np.array_equal(mx, kmax[s:s + 1])
    dv = oracle.dense_prefix_varlen(sh, lens, x["Qp"], x["K"], x["V"], x["Kb"], x["Vb"])
    for key in cache:
        assert np.array_equal(dv[key], cache[key]), key
    r = oracle.step(sh, x["Qc"], x["Qp"], x["K"], x["V"], kmin, kmax, x["Kb"], x["Vb"],
                    cache["o_p"], cache["l_p"])
    rv = oracle.step_varlen(sh, lens, x["Qc"], x["Qp"], x["K"], x["V"], x["Kb"], x["Vb"],
                            cache["o_p"], cache["l_p"])
    for key in rv:
        assert np.array_equal(rv[key], r[key]), key


def pin_varlen_short_sequences():
    """Sequences of different lengths (NaN past each): every value is finite;
    the dense pass is numpy attention over each sequence's own tokens; a
    sequence shorter than the budget selects all of its pages (its active rows'
    o_p is then its dense prefix attention) with the page lists padded by -1;
    a one-token prefix attends to that token alone (o_p = its value row)."""
    rng = np.random.default_rng(32)
    sh = rand_shape(rng, S=3, L=45, ps=4, B=6, A=2, budget=12)  # k = 3 pages
    x = rand_inputs(rng, sh)
    lens = [45, 7, 1]
    K, V = x["K"].copy(), x["V"].copy()
    for s, L in enumerate(lens):
        K[s, :, L:] = np.nan
        V[s, :, L:] = np.nan
    G = sh.Hq // sh.Hkv
    cache = oracle.dense_prefix_varlen(sh, lens, x["Qp"], K, V, x["Kb"], x["Vb"])
    for key in cache:
        assert np.isfinite(cache[key]).all(), key
    for s, L in enumerate(lens):
        for h in range(sh.Hq):
            for t in range(sh.B):
                o, l = np_attend(x["Qp"][s, h, t], K[s, h // G, :L], V[s, h // G, :L], sh.scale)
                close(cache["o_p"][s, h, t], o, 1e-6, "varlen dense o_p")
                close(cache["l_p"][s, h, t], l, 1e-5, "varlen dense L_p")
    r = oracle.step_varlen(sh, lens, x["Qc"], x["Qp"], K, V, x["Kb"], x["Vb"],
                           cache["o_p"], cache["l_p"])
    for key in ("o_p", "l_p", "out", "lse"):
        assert np.isfinite(r[key]).all(), key
    assert r["page_idx"].shape[-1] == 3
    assert np.all(r["page_idx"][1] == np.array([0, 1, -1])), "7 tokens: both pages, then -1"
    assert np.all(r["page_idx"][2] == np.array([0, -1, -1])), "1 token: page 0, then -1"
    assert np.all(r["union_count"][1] == 2) and np.all(r["union_count"][2] == 1)
    for s, L in ((1, 7), (2, 1)):
        for h in range(sh.Hq):
            for t in r["active_idx"][s, h]:
                o, l = np_attend(x["Qc"][s, h, t], K[s, h // G, :L], V[s, h // G, :L], sh.scale)
                close(r["o_p"][s, h, t], o, 1e-6, "short sequence: dense over its tokens")
                if L == 1:
                    close(r["o_p"][s, h, t], V[s, h // G, 0], 1e-6, "one token: its value")
    s0 = oracle.seq_shape(sh, 45)
    kmin, kmax = oracle.build_meta(s0, x["K"][:1])
    alone = oracle.step(s0, x["Qc"][:1], x["Qp"][:1], x["K"][:1], x["V"][:1], kmin, kmax,
                        x["Kb"][:1], x["Vb"][:1], cache["o_p"][:1], cache["l_p"][:1])
    for key in alone:
        assert np.array_equal(r[key][:1], alone[key]), key


def pin_varlen_append():
    """Each sequence's block lands at its own length (bitwise concatenation)."""
    rng = np.random.default_rng(33)
    f = lambda *s_: rng.standard_normal(s_).astype(np.float32)
    K, V, Kb, Vb = f(3, 2, 20, 8), f(3, 2, 20, 8), f(3, 2, 5, 8), f(3, 2, 5, 8)
    lens = [20, 9, 1]
    for s, (K2, V2) in enumerate(oracle.append_block_varlen(lens, K, V, Kb, Vb)):
        L = lens[s]
        assert K2.shape == (1, 2, L + 5, 8)
        assert np.array_equal(K2[0, :, :L], K[s, :, :L]) and np.array_equal(K2[0, :, L:], Kb[s])
        assert np.array_equal(V2[0, :, :L], V[s, :, :L]) and np.array_equal(V2[0, :, L:], Vb[s])


PINS = [v for n, v in sorted(globals().items()) if n.startswith("pin_")]
