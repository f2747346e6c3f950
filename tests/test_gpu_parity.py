"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs, on every workload and on edge-case shapes."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from losa_testutil import (DEV, TOL, Case, check_meta, check_step_full, check_step_sampled,
                           gpu_dense, gpu_meta, gpu_step, maxabs, oshape, random_case)
from sparse_long_context_mse_b200 import api, synth

pytestmark = pytest.mark.gpu


def clone_cache(d):
    return {"o_p": d["o_p"].clone(), "l_p": d["l_p"].clone()}


# ---------------------------------------------------------------------------
# page metadata: bit-exact
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [synth.TINY, synth.GQA16K, synth.GQA64K, synth.BATCH8])
def test_meta_exact(w):
    c = Case(synth.workload(w), gen_device="cpu" if w in (synth.TINY, synth.GQA16K) else DEV)
    meta = gpu_meta(c.sh, c.K)
    check_meta(c.sh, meta, c.host("K"))


def test_meta_exact_stack_layer():
    c = Case(synth.workload(synth.STACK36), layer=35, gen_device=DEV)
    meta = gpu_meta(c.sh, c.K)
    check_meta(c.sh, meta, c.host("K"))


# ---------------------------------------------------------------------------
# cold-start dense pass
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [synth.TINY, synth.GQA16K])
def test_dense_full(w):
    c = Case(synth.workload(w))
    g = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    o = oracle.dense_prefix(oshape(c.sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    for k in ("o_p", "l_p", "out", "lse"):
        e = maxabs(g[k].cpu().numpy(), o[k])
        assert e <= TOL, (k, e)


@pytest.mark.parametrize("w", [synth.GQA64K, synth.BATCH8])
def test_dense_sampled(w):
    c = Case(synth.workload(w), gen_device=DEV)
    g = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    sh = c.sh
    osh = oshape(sh)
    nrows = sh.num_seqs * sh.n_q_heads * sh.block_size
    rows = np.random.default_rng({synth.GQA64K: 2, synth.BATCH8: 3}[w]).choice(nrows, size=32,
                                                                          replace=False)
    o_d, l_d = oracle.dense_rows(osh, c.q[0], c.host("K"), c.host("V"), rows)
    gp = g["o_p"].reshape(nrows, -1).cpu().numpy()
    gl = g["l_p"].reshape(nrows).cpu().numpy()
    go = g["out"].reshape(nrows, -1).cpu().numpy()
    Q = oracle.f32(c.q[0]).reshape(nrows, -1)
    Kb, Vb = oracle.f32(c.kb[0]), oracle.f32(c.vb[0])
    for n_, r in enumerate(rows):
        assert maxabs(gp[r], o_d[n_]) <= TOL
        assert abs(gl[r] - l_d[n_]) <= TOL
        s, h = r // (sh.n_q_heads * sh.block_size), (r // sh.block_size) % sh.n_q_heads
        g_ = h // sh.group
        os_, ls = oracle.attend_tokens(Q[r], Kb[s, g_], Vb[s, g_], np.arange(sh.block_size),
                                       sh.scale)
        om, _ = oracle.merge(o_d[n_].astype(np.float64), float(l_d[n_]), os_, ls)
        assert maxabs(go[r], om) <= TOL


# ---------------------------------------------------------------------------
# one LoSA step
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("w", [synth.TINY, synth.GQA16K])
def test_step_full(w):
    c = Case(synth.workload(w))
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache_g["o_p"].clone(), cache_g["l_p"].clone())
    _, errs, exact = check_step_full(c, 1, res, cache_o, kmin, kmax, tag=w)
    # stable rows untouched
    act = res["active_idx"].cpu().numpy()
    for s in range(sh.num_seqs):
        for h in range(sh.n_q_heads):
            st = [t for t in range(sh.block_size) if t not in set(act[s, h].tolist())]
            assert torch.equal(res["o_p"][s, h, st], cache_g["o_p"][s, h, st])
            assert torch.equal(res["l_p"][s, h, st], cache_g["l_p"][s, h, st])
    # planted actives recovered exactly
    assert np.array_equal(act, np.stack([np.stack([np.nonzero(c.planted[0][s, h].numpy())[0]
                                                   for h in range(sh.n_q_heads)])
                                         for s in range(sh.num_seqs)]))
    assert api.read_device_status(res["ws"]) == api.LOSA_OK


@pytest.mark.parametrize("w,layer", [(synth.GQA64K, 0), (synth.BATCH8, 0), (synth.STACK36, 0),
                                     (synth.STACK36, 17), (synth.STACK36, 35)])
def test_step_sampled(w, layer):
    c = Case(synth.workload(w), layer=layer, gen_device=DEV)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_in = clone_cache(cache_g)
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], cache_g["o_p"],
                   cache_g["l_p"])
    check_step_sampled(c, 1, res, cache_in, kmin, kmax, tag=f"{w}/L{layer}")
    assert api.read_device_status(res["ws"]) == api.LOSA_OK


# ---------------------------------------------------------------------------
# step variants
# ---------------------------------------------------------------------------
def _union_case(name):
    if name in (synth.TINY, synth.GQA16K):
        return Case(synth.workload(name))
    if name == "groups_bf16":
        return random_case(2, 8, 2, 1000, 16, 4, 64, "bf16", seed=5)
    return random_case(1, 4, 1, 777, 8, 3, 48, "f32", seed=6)


@pytest.mark.parametrize("name", [synth.TINY, synth.GQA16K, "groups_bf16", "ragged_f32"])
def test_step_attend_union(name):
    """Every active row attends to its group's whole page union: the
    selection is the plain step's, o_p/L_p/out are the oracle's union
    attention."""
    c = _union_case(name)
    c.sh.flags = api.LOSA_STEP_ATTEND_UNION
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache_g["o_p"].clone(), cache_g["l_p"].clone())
    ref, _, _ = check_step_full(c, 1, res, cache_o, kmin, kmax, tag=f"union {name}")
    # the union rows differ from the plain step's wherever the union added pages
    sh.flags = 0
    plain = oracle.step_forced(oshape(sh), c.q[1], c.host("K"), c.host("V"), c.kb[1], c.vb[1],
                               res["active_idx"].cpu().numpy(), res["page_idx"].cpu().numpy(),
                               cache_o["o_p"], cache_o["l_p"])
    if sh.n_active * sh.group > 1 and sh.pages_per_row < sh.n_pages:
        assert maxabs(ref["l_p"], plain["l_p"]) > 10 * TOL, "the case does not exercise the union"
    assert api.read_device_status(res["ws"]) == api.LOSA_OK


@pytest.mark.parametrize("w", [synth.TINY, synth.GQA16K])
def test_step_ref_chain(w):
    """Drift-safe locality over a denoising chain: each step scores against
    the reference queries, the GPU's reference is rewritten exactly for the
    active rows, and every output matches the oracle's drift-safe step."""
    cfg = synth.workload(w)
    T = 4
    c = Case(cfg, steps=T)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    q_ref_g = c.q[0].clone()
    q_ref_o = oracle.f32(c.q[0])
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, DEV)
    for t in range(1, T):
        res = gpu_step(sh, c.q[t], None, c.K, c.V, meta, c.kb[t], c.vb[t], cache_g["o_p"],
                       cache_g["l_p"], ws=ws, q_ref=q_ref_g)
        ref, _, _ = check_step_full(c, t, res, cache_o, kmin, kmax, tag=f"ref {w} t{t}",
                                    qp=q_ref_o)
        q_ref_o = oracle.refresh_ref(oshape(sh), c.q[t], res["active_idx"].cpu().numpy(), q_ref_o)
        assert np.array_equal(oracle.f32(q_ref_g).view(np.uint32), q_ref_o.view(np.uint32)), t
        cache_o = {"o_p": ref["o_p"], "l_p": ref["l_p"]}
    assert api.read_device_status(ws) == api.LOSA_OK


# ---------------------------------------------------------------------------
# denoising chains: step 1 dense, then LoSA steps, cache carried through
# ---------------------------------------------------------------------------
def test_chain_full_16k():
    cfg = synth.workload(synth.GQA16K)
    T = 4
    c = Case(cfg, steps=T)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, DEV)
    for t in range(1, T):
        res = gpu_step(sh, c.q[t], c.q[t - 1], c.K, c.V, meta, c.kb[t], c.vb[t],
                       cache_g["o_p"], cache_g["l_p"], ws=ws)
        ref, _, _ = check_step_full(c, t, res, cache_o, kmin, kmax, tag=f"chain1 t{t}")
        cache_o = {"o_p": ref["o_p"], "l_p": ref["l_p"]}


def test_chain_sampled_64k():
    cfg = synth.workload(synth.GQA64K)
    T = cfg.steps
    c = Case(cfg, steps=T, gen_device=DEV)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, DEV)
    for t in range(1, T):
        cache_in = clone_cache(cache_g)
        res = gpu_step(sh, c.q[t], c.q[t - 1], c.K, c.V, meta, c.kb[t], c.vb[t],
                       cache_g["o_p"], cache_g["l_p"], ws=ws)
        if t == 1:
            check_step_sampled(c, t, res, cache_in, kmin, kmax, tag=f"chain2 t{t}")
        else:
            # the cache of rows refreshed at earlier steps is sparse, not dense:
            # check active rows and the untouched stable rows only
            check_step_sampled(c, t, res, cache_in, kmin, kmax, n_stable=0, tag=f"chain2 t{t}")
    assert api.read_device_status(ws) == api.LOSA_OK


# ---------------------------------------------------------------------------
# edge cases (full oracle comparison)
# ---------------------------------------------------------------------------
EDGE = {
    # name: (S, Hq, Hkv, L, B, A, budget, dtype)
    "ragged_f32": (3, 6, 2, 1000, 5, 2, 48, "f32"),
    "ragged_bf16": (3, 6, 2, 1000, 5, 2, 48, "bf16"),
    "one_page": (1, 2, 1, 7, 3, 1, 16, "bf16"),
    "k1_many_pages": (1, 4, 2, 5000, 16, 3, 16, "bf16"),
    "k64": (1, 4, 1, 20000, 8, 2, 1024, "bf16"),
    "rows128": (1, 8, 1, 3000, 16, 16, 256, "bf16"),
    "B32_G4": (2, 8, 2, 2500, 32, 8, 256, "bf16"),
    "all_pages_big_k": (1, 4, 2, 1600, 16, 4, 1600, "bf16"),
    "zero_active": (2, 4, 2, 900, 16, 0, 128, "bf16"),
    "dense_equivalent": (1, 4, 2, 777, 16, 16, 1024, "f32"),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge(name):
    S, Hq, Hkv, L, B, A, budget, dt = EDGE[name]
    c = random_case(S, Hq, Hkv, L, B, A, budget, dt, seed=zlib.crc32(name.encode()) % 1000)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    for k in ("o_p", "l_p", "out", "lse"):
        assert maxabs(cache_g[k].cpu().numpy(), cache_o[k]) <= TOL, (name, "dense", k)
    cache_in = clone_cache(cache_g)
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], cache_g["o_p"],
                   cache_g["l_p"])
    check_step_full(c, 1, res, cache_o, kmin, kmax, tag=name)
    if A == 0:
        assert torch.equal(res["o_p"], cache_in["o_p"]) and torch.equal(res["l_p"], cache_in["l_p"])
        assert int(res["union_count"].abs().sum()) == 0
    if name == "dense_equivalent":
        dense_now = gpu_dense(sh, c.q[1], c.K, c.V, c.kb[1], c.vb[1])
        assert maxabs(res["out"].cpu().numpy(), dense_now["out"].cpu().numpy()) <= TOL
    assert api.read_device_status(res["ws"]) == api.LOSA_OK


@pytest.mark.parametrize("variant", ["union", "ref", "capacity"])
@pytest.mark.parametrize("name", ["ragged_bf16", "one_page", "rows128", "all_pages_big_k",
                                  "zero_active", "k64"])
def test_edge_variants(name, variant):
    """The edge shapes under each variant: attending to the whole union,
    drift-safe locality against a reference, prefix buffers with a capacity
    beyond the prefix (unaligned, never read)."""
    S, Hq, Hkv, L, B, A, budget, dt = EDGE[name]
    c = random_case(S, Hq, Hkv, L, B, A, budget, dt, seed=zlib.crc32((name + variant).encode()) % 1000)
    sh = c.sh
    Kh, Vh = c.host("K"), c.host("V")
    if variant == "union":
        sh.flags = api.LOSA_STEP_ATTEND_UNION
    if variant == "capacity":
        cap = L + 37
        K = torch.full((S, Hkv, cap, 128), 3.0, dtype=c.K.dtype, device=DEV)
        V = torch.full_like(K, -3.0)
        K[:, :, :L] = c.K
        V[:, :, :L] = c.V
        sh.prefix_capacity = cap
        c.K, c.V = K, V
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, Kh)
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], Kh, Vh, c.kb[0], c.vb[0])
    for k in ("o_p", "l_p", "out", "lse"):
        assert maxabs(cache_g[k].cpu().numpy(), cache_o[k]) <= TOL, (name, variant, "dense", k)
    q_ref = c.q[0].clone() + 0.25 if variant == "ref" else None
    if q_ref is not None:
        q_ref = q_ref.to(c.q[0].dtype)
        q_ref_o = oracle.f32(q_ref)
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], cache_g["o_p"],
                   cache_g["l_p"], q_ref=q_ref)
    check_step_full(c, 1, res, cache_o, kmin, kmax, tag=f"{name}/{variant}",
                    qp=q_ref_o if q_ref is not None else None)
    if q_ref is not None:
        want = oracle.refresh_ref(oshape(sh), c.q[1], res["active_idx"].cpu().numpy(), q_ref_o)
        assert np.array_equal(oracle.f32(q_ref).view(np.uint32), want.view(np.uint32))
    assert api.read_device_status(res["ws"]) == api.LOSA_OK


def test_deterministic():
    c = Case(synth.workload(synth.GQA16K))
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    cache = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    outs = []
    for _ in range(2):
        r = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                     cache["o_p"].clone(), cache["l_p"].clone())
        outs.append(r)
    for k in ("out", "lse", "o_p", "l_p", "active_idx", "page_idx", "union_count"):
        assert torch.equal(outs[0][k], outs[1][k]), k


def test_python_binding_rejects_bad_tensors():
    c = random_case(1, 4, 2, 100, 16, 2, 32)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    cache = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    with pytest.raises(ValueError):
        gpu_step(sh, c.q[1].float(), c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                 cache["o_p"], cache["l_p"])
    with pytest.raises(ValueError):
        gpu_step(sh, c.q[1].cpu(), c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                 cache["o_p"], cache["l_p"])
