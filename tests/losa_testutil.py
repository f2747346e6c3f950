"""Helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same seeded inputs, compare.

The comparison rules:
  * page metadata, active sets, page lists and union counts: bit-exact, with
    no tolerance at all -- the CUDA path takes the oracle's decisions exactly
    (locality in the oracle's channel order; page bounds with a proven error
    interval and exact rescoring wherever the interval leaves the top k open),
    ties included;
  * prefix outputs o_p, log-normalisers L_p, outputs and their lse: max-abs
    error <= 2e-3 (bf16 or fp32 K/V, fp32 accumulation);
  * stable rows of the cache: bitwise untouched by the step.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from sparse_long_context_mse_b200 import api, synth

DEV = "cuda:0"
TOL = 2e-3


def scale_of(d):
    return float(np.float32(1.0 / np.sqrt(d)))


def unswizzle_page_meta(sh, page_meta):
    """(kmin, kmax) ``[S][Hkv][P][d]`` from the library's documented layout:
    record (s*Hkv+g)*P + p holds kmin then kmax; logical 16-byte chunk c sits
    at chunk c ^ (p & 7).  Pure index permutation."""
    esz = 2 if sh.dtype == api.LOSA_BF16 else 4
    P, d = sh.n_pages, sh.head_dim
    Pc = (sh.capacity + sh.page_size - 1) // sh.page_size  # records per (s, g)
    nchunk = 2 * d * esz // 16
    nrec = sh.num_seqs * sh.n_kv_heads * Pc
    raw = page_meta.detach().cpu().view(torch.uint8)[:nrec * nchunk * 16].reshape(
        sh.num_seqs * sh.n_kv_heads, Pc, nchunk, 16)[:, :P]
    pages = torch.arange(P)
    phys = torch.arange(nchunk)[None, :] ^ (pages[:, None] & 7)
    idx = phys[None, :, :, None].expand(raw.shape[0], P, nchunk, 16)
    logical = torch.gather(raw, 2, idx).reshape(-1).view(sh.torch_dtype)
    logical = logical.reshape(sh.num_seqs, sh.n_kv_heads, P, 2, d)
    return logical[:, :, :, 0].contiguous(), logical[:, :, :, 1].contiguous()


def oshape(sh):
    flags = oracle.ATTEND_UNION if sh.flags & api.LOSA_STEP_ATTEND_UNION else 0
    return oracle.shape(sh.num_seqs, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, sh.prefix_len,
                        sh.page_size, sh.block_size, sh.n_active, sh.token_budget, sh.scale,
                        flags)


def maxabs(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.max(np.abs(a - b))) if a.size else 0.0


# ---------------------------------------------------------------------------
# inputs
# ---------------------------------------------------------------------------
class Case:
    """Seeded inputs of one layer of a workload, resident on the GPU."""

    def __init__(self, cfg, layer=0, steps=2, gen_device="cpu"):
        self.cfg = cfg.for_layer(layer)
        self.layer = layer
        self.sh = api.shape_of(self.cfg, scale=scale_of(self.cfg.head_dim))
        pre = synth.gen_prefix(cfg, layer, device=gen_device)
        self.K = pre["k_prefix"].to(DEV)
        self.V = pre["v_prefix"].to(DEV)
        q = synth.gen_queries(self.cfg, layer, steps=steps, device=gen_device,
                              hot_u=pre["hot_u"])
        self.q = [t.to(DEV) for t in q["q"]]
        self.planted = q["planted"]
        self.kb, self.vb = [], []
        for t in range(steps):
            a, b = synth.gen_block_kv(cfg, layer, t, device=gen_device)
            self.kb.append(a.to(DEV))
            self.vb.append(b.to(DEV))
        self._host = {}

    def host(self, name):
        """fp32 numpy copy (cached) of a GPU tensor attribute."""
        if name not in self._host:
            self._host[name] = oracle.f32(getattr(self, name))
        return self._host[name]


def random_case(S, Hq, Hkv, L, B, A, budget, dtype="bf16", seed=0, drift_active=1.0,
                drift_stable=0.01):
    """Plain random inputs for edge-case shapes (same recipe, no hot pages)."""
    g = torch.Generator().manual_seed(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = 128
    r = lambda *s: torch.randn(*s, generator=g)
    qp = r(S, Hq, B, d)
    drift = r(S, Hq, B, d)
    sig = torch.full((S, Hq, B), drift_stable)
    for s in range(S):
        for h in range(Hq):
            sig[s, h, torch.randperm(B, generator=g)[:A]] = drift_active
    qc = qp + sig[..., None] * drift
    c = Case.__new__(Case)
    c.cfg = None
    c.layer = 0
    c.sh = api.make_shape(S, Hq, Hkv, d, L, 16, B, A, budget, dtype, scale=scale_of(d))
    c.K = r(S, Hkv, L, d).to(tdt).to(DEV)
    c.V = r(S, Hkv, L, d).to(tdt).to(DEV)
    c.q = [qp.to(tdt).to(DEV), qc.to(tdt).to(DEV)]
    c.kb = [r(S, Hkv, B, d).to(tdt).to(DEV) for _ in range(2)]
    c.vb = [r(S, Hkv, B, d).to(tdt).to(DEV) for _ in range(2)]
    c.planted = None
    c._host = {}
    return c


# ---------------------------------------------------------------------------
# GPU path (through the C ABI)
# ---------------------------------------------------------------------------
def gpu_meta(sh, K):
    meta = api.alloc_page_meta(sh, DEV)
    api.build_page_meta(sh, K, meta)
    return meta


def gpu_dense(sh, q, K, V, kb, vb, ws=None):
    rows = (sh.num_seqs, sh.n_q_heads, sh.block_size)
    o_p = torch.empty(*rows, sh.head_dim, device=DEV)
    l_p = torch.empty(*rows, device=DEV)
    out = torch.empty_like(o_p)
    lse = torch.empty_like(l_p)
    if ws is None:
        ws = api.alloc_workspace(sh, api.LOSA_WS_DENSE, DEV)
    api.dense_prefix(sh, q, K, V, kb, vb, o_p, l_p, out, lse, ws)
    return {"o_p": o_p, "l_p": l_p, "out": out, "lse": lse}


def gpu_step(sh, qc, qp, K, V, meta, kb, vb, o_p, l_p, ws=None, q_ref=None):
    """One step; o_p/l_p are updated in place (pass clones to keep inputs).
    With ``q_ref`` (drift-safe locality) ``qp`` is ignored and ``q_ref`` is
    the in/out reference."""
    rows = (sh.num_seqs, sh.n_q_heads, sh.block_size)
    out = torch.empty(*rows, sh.head_dim, device=DEV)
    lse = torch.empty(*rows, device=DEV)
    A, k = sh.n_active, sh.pages_per_row
    act = torch.full((sh.num_seqs, sh.n_q_heads, A), -7, dtype=torch.int32, device=DEV)
    pidx = torch.full((sh.num_seqs, sh.n_q_heads, A, k), -7, dtype=torch.int32, device=DEV)
    uc = torch.full((sh.num_seqs, sh.n_kv_heads), -7, dtype=torch.int32, device=DEV)
    if ws is None:
        ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, DEV)
    if q_ref is None:
        api.step(sh, qc, qp, K, V, meta, kb, vb, o_p, l_p, out, lse, ws, act, pidx, uc)
    else:
        api.step_ref(sh, qc, q_ref, K, V, meta, kb, vb, o_p, l_p, out, lse, ws, act, pidx, uc)
    return {"out": out, "lse": lse, "o_p": o_p, "l_p": l_p, "active_idx": act,
            "page_idx": pidx, "union_count": uc, "ws": ws}


# ---------------------------------------------------------------------------
# comparisons
# ---------------------------------------------------------------------------
def page_norms(sh, page_meta):
    """The metadata's page-norm rows ``[S][Hkv][P][2]`` (||kmin||, ||kmax||):
    after the records, float2 per page, rows padded to a multiple of 8 pages."""
    esz = 2 if sh.dtype == api.LOSA_BF16 else 4
    P, d = sh.n_pages, sh.head_dim
    Pc = (sh.capacity + sh.page_size - 1) // sh.page_size
    Pn = (Pc + 7) // 8 * 8
    nrec = sh.num_seqs * sh.n_kv_heads * Pc
    raw = page_meta.detach().cpu().view(torch.uint8)[nrec * 2 * d * esz:]
    nrm = raw[:sh.num_seqs * sh.n_kv_heads * Pn * 8].view(torch.float32)
    return nrm.reshape(sh.num_seqs, sh.n_kv_heads, Pn, 2)[:, :, :P].numpy()


def check_meta(sh, meta, K_host):
    kmin_g, kmax_g = unswizzle_page_meta(sh, meta)
    kmin_o, kmax_o = oracle.build_meta(oshape(sh), K_host)
    assert np.array_equal(kmin_g.float().numpy().view(np.uint32), kmin_o.view(np.uint32))
    assert np.array_equal(kmax_g.float().numpy().view(np.uint32), kmax_o.view(np.uint32))
    # the page norms bound the exact norms of the (exact) records from above,
    # and closely: fp32 sums of 128 squares with every rounding upward
    nrm = page_norms(sh, meta).astype(np.float64)
    for j, m in enumerate((kmin_o, kmax_o)):
        exact = np.sqrt(np.sum(np.asarray(m, np.float64) ** 2, axis=-1))
        assert np.all(nrm[..., j] >= exact)
        assert np.all(nrm[..., j] <= exact * (1 + 2.0 ** -15) + 1e-30)
    return kmin_o, kmax_o


def _boundary_gap(scores, n):
    """Relative gap between the n-th and (n+1)-th largest score."""
    if n <= 0 or n >= len(scores):
        return np.inf
    srt = np.sort(np.asarray(scores, np.float64))[::-1]
    return (srt[n - 1] - srt[n]) / max(abs(srt[n - 1]), 1e-30)


def check_step_sampled(c, step_t, res, cache_in, kmin, kmax, n_stable=24, rng_seed=0, tag=""):
    """Compare one GPU step with the oracle, computing the oracle row by row:
    every active row in full, plus a sample of stable rows."""
    sh = c.sh
    osh = oshape(sh)
    G = sh.group
    k = sh.pages_per_row
    Qc = oracle.f32(c.q[step_t])
    Qp = oracle.f32(c.q[step_t - 1])
    Kh, Vh = c.host("K"), c.host("V")
    Kb = oracle.f32(c.kb[step_t])
    Vb = oracle.f32(c.vb[step_t])
    mse = oracle.locality(osh, Qc, Qp)
    act_o = oracle.active(osh, mse)
    act_g = res["active_idx"].cpu().numpy()
    pidx_g = res["page_idx"].cpu().numpy()
    uc_g = res["union_count"].cpu().numpy()
    o_p_g = res["o_p"].cpu().numpy()
    l_p_g = res["l_p"].cpu().numpy()
    out_g = res["out"].cpu().numpy()
    lse_g = res["lse"].cpu().numpy()
    cache_o = cache_in["o_p"].cpu().numpy()
    cache_l = cache_in["l_p"].cpu().numpy()
    err = {"o_p": 0.0, "l_p": 0.0, "out": 0.0, "lse": 0.0}
    for s in range(sh.num_seqs):
        unions = [set() for _ in range(sh.n_kv_heads)]
        for h in range(sh.n_q_heads):
            g = h // G
            assert np.array_equal(act_o[s, h], act_g[s, h]), (
                f"{tag} active set differs at s{s} h{h}: gpu {act_g[s, h]} oracle {act_o[s, h]} "
                f"(boundary gap {_boundary_gap(mse[s, h], sh.n_active):.3g})")
            for a in range(sh.n_active):
                t = int(act_g[s, h, a])
                if sh.pages_per_row == sh.n_pages:
                    pages_o = np.arange(sh.n_pages, dtype=np.int32)
                    U = None
                else:
                    U = oracle.bound_scores(Qc[s, h, t], kmin[s, g], kmax[s, g])
                    pages_o = oracle.topk_pages(U, k)
                pages = pages_o
                assert np.array_equal(pages_o, pidx_g[s, h, a]), (
                    f"{tag} pages differ at s{s} h{h} t{t}: gpu {pidx_g[s, h, a]} "
                    f"oracle {pages_o} (boundary gap {_boundary_gap(U, k):.3g})")
                unions[g].update(int(p) for p in pages)
                tok = np.concatenate([np.arange(p * 16, min(p * 16 + 16, sh.prefix_len))
                                      for p in pages]).astype(np.int32)
                o, L = oracle.attend_tokens(Qc[s, h, t], Kh[s, g], Vh[s, g], tok, sh.scale)
                err["o_p"] = max(err["o_p"], maxabs(o_p_g[s, h, t], o))
                err["l_p"] = max(err["l_p"], abs(float(l_p_g[s, h, t]) - L))
                os_, ls = oracle.attend_tokens(Qc[s, h, t], Kb[s, g], Vb[s, g],
                                               np.arange(sh.block_size), sh.scale)
                om, lm = oracle.merge(np.float32(o).astype(np.float64), float(np.float32(L)),
                                      os_, ls)
                err["out"] = max(err["out"], maxabs(out_g[s, h, t], om))
                err["lse"] = max(err["lse"], abs(float(lse_g[s, h, t]) - lm))
        for g in range(sh.n_kv_heads):
            assert uc_g[s, g] == len(unions[g]), f"{tag} union count s{s} g{g}"
    # stable rows: bitwise untouched cache, out = merge(cache, suffix)
    rng = np.random.default_rng(rng_seed)
    stable = [(s, h, t) for s in range(sh.num_seqs) for h in range(sh.n_q_heads)
              for t in range(sh.block_size) if t not in set(act_g[s, h].tolist())]
    for s, h, t in stable:
        assert np.array_equal(o_p_g[s, h, t].view(np.uint32), cache_o[s, h, t].view(np.uint32))
        assert l_p_g[s, h, t].view(np.uint32) == cache_l[s, h, t].view(np.uint32)
    pick = rng.choice(len(stable), size=min(n_stable, len(stable)), replace=False) if stable else []
    rows = [((s * sh.n_q_heads + h) * sh.block_size + t) for s, h, t in (stable[i] for i in pick)]
    if rows:
        o_d, l_d = oracle.dense_rows(osh, Qp, Kh, Vh, rows)
        for n, i in enumerate(pick):
            s, h, t = stable[i]
            g = h // G
            err["o_p"] = max(err["o_p"], maxabs(cache_o[s, h, t], o_d[n]))
            err["l_p"] = max(err["l_p"], abs(float(cache_l[s, h, t]) - float(l_d[n])))
            os_, ls = oracle.attend_tokens(Qc[s, h, t], Kb[s, g], Vb[s, g],
                                           np.arange(sh.block_size), sh.scale)
            om, lm = oracle.merge(o_d[n].astype(np.float64), float(l_d[n]), os_, ls)
            err["out"] = max(err["out"], maxabs(out_g[s, h, t], om))
            err["lse"] = max(err["lse"], abs(float(lse_g[s, h, t]) - lm))
    for key, v in err.items():
        assert v <= TOL, f"{tag} {key} max-abs err {v:.3g} > {TOL}"
    return err


def check_step_full(c, step_t, res, cache_o_in, kmin, kmax, tag="", qp=None):
    """Compare every output of one GPU step with the oracle's full step run on
    the oracle's own cache (``cache_o_in``: dict from oracle.dense_prefix or a
    previous oracle.step).  ``qp``: the locality reference (default: the
    previous step's queries)."""
    sh = c.sh
    osh = oshape(sh)
    qp = c.q[step_t - 1] if qp is None else qp
    r = oracle.step(osh, c.q[step_t], qp, c.host("K"), c.host("V"), kmin, kmax,
                    c.kb[step_t], c.vb[step_t], cache_o_in["o_p"], cache_o_in["l_p"],
                    want_bound=sh.pages_per_row < sh.n_pages)
    act_g = res["active_idx"].cpu().numpy()
    pidx_g = res["page_idx"].cpu().numpy()
    for s in range(sh.num_seqs):
        for h in range(sh.n_q_heads):
            assert np.array_equal(act_g[s, h], r["active_idx"][s, h]), (
                f"{tag} active set differs s{s} h{h}: gpu {act_g[s, h]} oracle "
                f"{r['active_idx'][s, h]} (gap {_boundary_gap(r['mse'][s, h], sh.n_active):.3g})")
            for a in range(sh.n_active):
                gap = (_boundary_gap(r["bound"][s, h, a], sh.pages_per_row)
                       if "bound" in r and r["bound"] is not None else float("nan"))
                assert np.array_equal(pidx_g[s, h, a], r["page_idx"][s, h, a]), (
                    f"{tag} pages differ s{s} h{h} a{a}: gpu {pidx_g[s, h, a]} oracle "
                    f"{r['page_idx'][s, h, a]} (gap {gap:.3g})")
    assert np.array_equal(res["union_count"].cpu().numpy(), r["union_count"]), tag
    ref = r
    exact_sel = True
    errs = {k: maxabs(res[k].cpu().numpy(), ref[k]) for k in ("o_p", "l_p", "out", "lse")}
    for key, v in errs.items():
        assert v <= TOL, f"{tag} {key} max-abs err {v:.3g} > {TOL}"
    return ref, errs, exact_sel
