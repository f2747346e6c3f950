"""Variable-length batches on the GPU: losa_shape.prefix_lens gives every
sequence its own prefix length inside capacity-strided buffers.  Each
sequence must match the oracle's one-sequence problem at its own length
(page lists padded with -1), whatever the buffers hold past that length:
the tails here are NaN, so a kernel that reads one shows it."""
import numpy as np
import pytest
import torch

import oracle
from losa_testutil import (DEV, TOL, check_step_full, gpu_dense, gpu_step, maxabs,
                           random_case, unswizzle_page_meta)
from sparse_long_context_mse_b200 import api

pytestmark = pytest.mark.gpu

# a full-length sequence, one shorter than the 4-page budget, a single token
# and a ragged one; the capacity is not a multiple of the page size
LENS = [1000, 37, 1, 513]
LC = 1003
META_FILL = 0x5A


class _Seq:
    """One sequence of a variable-length case, as a one-sequence case."""

    def __init__(self, c, s):
        L = c.lens[s]
        sh = c.sh
        self.sh = api.make_shape(1, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, L, sh.page_size,
                                 sh.block_size, sh.n_active, sh.token_budget, sh.dtype,
                                 scale=sh.scale, flags=sh.flags)
        self.q = [q[s:s + 1] for q in c.q]
        self.kb = [x[s:s + 1] for x in c.kb]
        self.vb = [x[s:s + 1] for x in c.vb]
        self._host = {"K": oracle.f32(c.K[s:s + 1, :, :L]), "V": oracle.f32(c.V[s:s + 1, :, :L])}

    def host(self, name):
        return self._host[name]


def _varlen_case(dtype, lens=LENS, Lc=LC, seed=0, A=4, budget=64, flags=0):
    S, Hq, Hkv, B, d = len(lens), 8, 2, 16, 128
    L = max(lens)
    c = random_case(S, Hq, Hkv, L, B, A, budget, dtype, seed=seed)
    K = torch.full((S, Hkv, Lc, d), float("nan"), dtype=c.K.dtype, device=DEV)
    V = torch.full_like(K, float("nan"))
    for s, Ls in enumerate(lens):
        K[s, :, :Ls] = c.K[s, :, :Ls]
        V[s, :, :Ls] = c.V[s, :, :Ls]
    c.lens = list(lens)
    c.lens_t = torch.tensor(lens, dtype=torch.int32, device=DEV)
    c.sh = api.make_shape(S, Hq, Hkv, d, L, 16, B, A, budget, dtype, scale=c.sh.scale,
                          flags=flags, prefix_capacity=Lc, prefix_lens=c.lens_t)
    c.K, c.V = K, V
    return c


def _meta(c):
    meta = api.alloc_page_meta(c.sh, DEV)
    meta.view(torch.uint8).fill_(META_FILL)
    api.build_page_meta(c.sh, c.K, meta)
    return meta


def _check_meta(c, meta):
    """Records of each sequence's own pages bit-exact against the oracle's
    build at its length; records past them never written."""
    sh = c.sh
    kmin_g, kmax_g = unswizzle_page_meta(sh, meta)
    ref = oracle.build_meta_varlen(oracle.shape(sh.num_seqs, sh.n_q_heads, sh.n_kv_heads, 128,
                                                sh.prefix_len, 16, sh.block_size, sh.n_active,
                                                sh.token_budget, sh.scale), c.lens, c.K)
    Pc = (sh.capacity + 15) // 16
    esz = 2 if sh.dtype == api.LOSA_BF16 else 4
    nrec = sh.num_seqs * sh.n_kv_heads * Pc
    raw = meta.view(torch.uint8)[:nrec * 2 * 128 * esz].reshape(
        sh.num_seqs * sh.n_kv_heads, Pc, -1).cpu()
    # the page norms: upper bounds of the records' exact norms, close to them;
    # entries past a sequence's pages never written
    Pn = (Pc + 7) // 8 * 8
    nrm_raw = meta.view(torch.uint8)[nrec * 2 * 128 * esz:].cpu()
    nrm = nrm_raw.view(torch.float32).reshape(sh.num_seqs, sh.n_kv_heads, Pn, 2).numpy()
    nrm_bytes = nrm_raw.reshape(sh.num_seqs, sh.n_kv_heads, Pn, 8)
    per_seq = []
    for s, (kmin_o, kmax_o) in enumerate(ref):
        P = kmin_o.shape[2]
        assert np.array_equal(kmin_g[s:s + 1, :, :P].float().numpy().view(np.uint32),
                              kmin_o.view(np.uint32)), s
        assert np.array_equal(kmax_g[s:s + 1, :, :P].float().numpy().view(np.uint32),
                              kmax_o.view(np.uint32)), s
        rows = raw[s * sh.n_kv_heads:(s + 1) * sh.n_kv_heads, P:]
        assert bool((rows == META_FILL).all()), f"records past sequence {s}'s pages written"
        for j, m in enumerate((kmin_o, kmax_o)):
            exact = np.sqrt(np.sum(np.asarray(m[0], np.float64) ** 2, axis=-1))
            got = nrm[s, :, :P, j].astype(np.float64)
            assert np.all(got >= exact) and np.all(got <= exact * (1 + 2.0 ** -15) + 1e-30), s
        assert bool((nrm_bytes[s, :, P:] == META_FILL).all()), f"norms past sequence {s}'s pages"
        per_seq.append((kmin_o, kmax_o))
    return per_seq


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_varlen_meta(dtype):
    c = _varlen_case(dtype, seed=1)
    _check_meta(c, _meta(c))


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_varlen_dense(dtype):
    c = _varlen_case(dtype, seed=2)
    ws_ok = api.alloc_workspace(c.sh, api.LOSA_WS_DENSE, DEV)
    got = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0], ws=ws_ok)
    osh = oracle.shape(c.sh.num_seqs, 8, 2, 128, c.sh.prefix_len, 16, 16, 4, 64, c.sh.scale)
    ref = oracle.dense_prefix_varlen(osh, c.lens, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    for key in ("o_p", "l_p", "out", "lse"):
        g = got[key].cpu().numpy()
        assert np.isfinite(g).all(), key
        assert maxabs(g, ref[key]) <= TOL, key
    assert api.read_device_status(ws_ok) == api.LOSA_OK


@pytest.mark.parametrize("dtype,flags", [("bf16", 0), ("f32", 0),
                                         ("bf16", api.LOSA_STEP_ATTEND_UNION)])
def test_varlen_step(dtype, flags):
    c = _varlen_case(dtype, seed=3, flags=flags)
    meta = _meta(c)
    per_meta = _check_meta(c, meta)
    cache = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    res = gpu_step(c.sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache["o_p"].clone(), cache["l_p"].clone())
    assert api.read_device_status(res["ws"]) == api.LOSA_OK
    k = c.sh.pages_per_row
    pidx = res["page_idx"].cpu().numpy()
    for s, L in enumerate(c.lens):
        sub = _Seq(c, s)
        ks = sub.sh.pages_per_row
        assert np.all(pidx[s, ..., ks:] == -1), f"sequence {s}: padding past its {ks} pages"
        one = {key: res[key][s:s + 1] for key in ("out", "lse", "o_p", "l_p", "active_idx",
                                                   "union_count")}
        one["page_idx"] = res["page_idx"][s:s + 1, ..., :ks]
        osh = oracle.seq_shape(oracle.shape(1, 8, 2, 128, L, 16, 16, 4, 64, c.sh.scale, flags), L)
        cache_o = oracle.dense_prefix(osh, c.q[0][s:s + 1], sub.host("K"), sub.host("V"),
                                      c.kb[0][s:s + 1], c.vb[0][s:s + 1])
        kmin, kmax = per_meta[s]
        check_step_full(sub, 1, one, cache_o, kmin, kmax, tag=f"varlen {dtype} s{s} L{L}")
    assert k == 4


def test_varlen_all_pages():
    # a budget covering the longest prefix: every sequence takes all of its
    # own pages, listed in order, then -1
    c = _varlen_case("bf16", seed=4, budget=1024)
    meta = _meta(c)
    cache = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    res = gpu_step(c.sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache["o_p"].clone(), cache["l_p"].clone())
    assert api.read_device_status(res["ws"]) == api.LOSA_OK
    k = c.sh.pages_per_row
    pidx = res["page_idx"].cpu().numpy()
    uc = res["union_count"].cpu().numpy()
    osh = oracle.shape(c.sh.num_seqs, 8, 2, 128, c.sh.prefix_len, 16, 16, 4, 1024, c.sh.scale)
    cache_o = oracle.dense_prefix_varlen(osh, c.lens, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    ref = oracle.step_varlen(osh, c.lens, c.q[1], c.q[0], c.K, c.V, c.kb[1], c.vb[1],
                             cache_o["o_p"], cache_o["l_p"])
    for s, L in enumerate(c.lens):
        P = (L + 15) // 16
        want = np.where(np.arange(k) < P, np.arange(k), -1)
        assert np.all(pidx[s] == want), s
        assert np.all(uc[s] == P), s
    assert np.array_equal(pidx, ref["page_idx"])
    assert np.array_equal(res["active_idx"].cpu().numpy(), ref["active_idx"])
    for key in ("o_p", "l_p", "out", "lse"):
        assert maxabs(res[key].cpu().numpy(), ref[key]) <= TOL, key


def test_varlen_equal_lengths_match_uniform_call():
    # every entry equal to prefix_len: bit-identical to the call without the array
    c = _varlen_case("bf16", lens=[700, 700, 700], Lc=700, seed=5)
    meta = _meta(c)
    cache = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    res = gpu_step(c.sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache["o_p"].clone(), cache["l_p"].clone())
    sh_u = api.make_shape(3, 8, 2, 128, 700, 16, 16, 4, 64, "bf16", scale=c.sh.scale)
    meta_u = api.alloc_page_meta(sh_u, DEV)
    api.build_page_meta(sh_u, c.K, meta_u)
    cache_u = gpu_dense(sh_u, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    res_u = gpu_step(sh_u, c.q[1], c.q[0], c.K, c.V, meta_u, c.kb[1], c.vb[1],
                     cache_u["o_p"].clone(), cache_u["l_p"].clone())
    torch.cuda.synchronize()
    # the written bytes agree: every record and every page's norms (the norm
    # rows' padding is never written)
    Pc = (700 + 15) // 16
    nrec_bytes = 3 * 2 * Pc * 2 * 128 * 2
    assert torch.equal(meta[:nrec_bytes], meta_u[:nrec_bytes])
    nrm = meta[nrec_bytes:].view(torch.float32).reshape(3, 2, -1, 2)[:, :, :Pc]
    nrm_u = meta_u[nrec_bytes:].view(torch.float32).reshape(3, 2, -1, 2)[:, :, :Pc]
    assert torch.equal(nrm, nrm_u)
    for key in ("o_p", "l_p", "out", "lse"):
        assert torch.equal(cache[key], cache_u[key]), key
    for key in ("out", "lse", "o_p", "l_p", "active_idx", "page_idx", "union_count"):
        assert torch.equal(res[key], res_u[key]), key


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_varlen_append(dtype):
    lens = [1000, 37, 1, 513]
    c = _varlen_case(dtype, lens=lens, Lc=1021, seed=6)
    meta = _meta(c)
    g = torch.Generator(device="cpu").manual_seed(66)
    kb = torch.randn(4, 2, 16, 128, generator=g).to(c.K.dtype).to(DEV)
    vb = torch.randn(4, 2, 16, 128, generator=g).to(c.K.dtype).to(DEV)
    grown = oracle.append_block_varlen(lens, c.K, c.V, kb, vb)
    api.append_block(c.sh, kb, vb, c.K, c.V, meta)
    torch.cuda.synchronize()
    c.lens = [L + 16 for L in lens]
    c.lens_t.copy_(torch.tensor(c.lens, dtype=torch.int32))
    c.sh.prefix_len += 16
    for s, (Ks, Vs) in enumerate(grown):
        L1 = c.lens[s]
        assert np.array_equal(oracle.f32(c.K[s:s + 1, :, :L1]).view(np.uint32), Ks.view(np.uint32))
        assert np.array_equal(oracle.f32(c.V[s:s + 1, :, :L1]).view(np.uint32), Vs.view(np.uint32))
        assert bool(torch.isnan(c.K[s, :, L1:].float()).all()), s  # the tail is not written
    # the rebuilt records equal a fresh build over the grown lengths; past a
    # sequence's new pages the records still hold what they held
    _check_meta(c, meta)


def test_varlen_entry_out_of_range_is_reported():
    # entries outside [1, prefix_len] are clamped (every access stays inside
    # the buffers) and reported through the device status
    c = _varlen_case("bf16", seed=7)
    meta = _meta(c)
    c.lens_t.copy_(torch.tensor([1000, 0, 1, 2000], dtype=torch.int32))
    ws_d = api.alloc_workspace(c.sh, api.LOSA_WS_DENSE, DEV)
    cache = gpu_dense(c.sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0], ws=ws_d)
    assert api.read_device_status(ws_d) == api.LOSA_ERR_DEVICE_BOUNDS
    res = gpu_step(c.sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache["o_p"].clone(), cache["l_p"].clone())
    assert api.read_device_status(res["ws"]) == api.LOSA_ERR_DEVICE_BOUNDS
    assert np.isfinite(res["out"][0].cpu().numpy()).all()
