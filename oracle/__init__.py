"""CPU oracle for LoSA per-denoising-step attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product (the CUDA library and its Python
binding) never imports it, and it imports nothing from the product.

The arithmetic lives in ``losa_oracle.c`` (plain C, compiled with
``-O2 -fno-fast-math -ffp-contract=off``); this module only builds that file
and marshals numpy arrays to it.  Every array argument is float32 (bf16
inputs are passed as their exact fp32 values) or int32, C-contiguous.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "losa_oracle.c")
_LIB = os.path.join(_HERE, "liblosa_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liblosa_oracle.so`` (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-std=c99",
                               "-Wall", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Shape(ctypes.Structure):
    _fields_ = [("S", ctypes.c_int), ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int),
                ("d", ctypes.c_int), ("L", ctypes.c_int), ("ps", ctypes.c_int),
                ("B", ctypes.c_int), ("A", ctypes.c_int), ("budget", ctypes.c_int),
                ("scale", ctypes.c_float), ("flags", ctypes.c_int)]


# variant bit: every active row attends to its GQA group's whole page union
ATTEND_UNION = 1


def shape(S, Hq, Hkv, d, L, ps, B, A, budget, scale=None, flags=0) -> Shape:
    if scale is None:
        scale = float(np.float32(1.0 / np.sqrt(d)))
    return Shape(S, Hq, Hkv, d, L, ps, B, A, budget, scale, flags)


def shape_of(cfg, scale=None, flags=0) -> Shape:
    return shape(cfg.num_seqs, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.prefix_len,
                 cfg.page_size, cfg.block_size, cfg.n_active, cfg.token_budget, scale, flags)


def _load():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.oracle_set_mutation.argtypes = [ctypes.c_int]
    return _lib


def _f(a):
    assert a.dtype == np.float32 and a.flags.c_contiguous, (a.dtype, a.flags)
    return a.ctypes.data_as(ctypes.c_void_p)


def _d(a):
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _i(a):
    assert a.dtype == np.int32 and a.flags.c_contiguous
    return a.ctypes.data_as(ctypes.c_void_p)


def _opt(a, conv):
    return None if a is None else conv(a)


def n_pages(sh: Shape) -> int:
    return (sh.L + sh.ps - 1) // sh.ps


def pages_per_row(sh: Shape) -> int:
    return min(sh.budget // sh.ps, n_pages(sh))


def set_mutation(m: int) -> None:
    """Plant deliberate bug number ``m`` (0 = none).  Tests only."""
    _load().oracle_set_mutation(int(m))


def f32(x) -> np.ndarray:
    """float32 C-contiguous numpy copy of a torch tensor or array."""
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.ascontiguousarray(x, dtype=np.float32)


def build_meta(sh: Shape, K):
    P = n_pages(sh)
    K = f32(K)
    kmin = np.empty((sh.S, sh.Hkv, P, sh.d), np.float32)
    kmax = np.empty_like(kmin)
    _load().oracle_build_meta(ctypes.byref(sh), _f(K), _f(kmin), _f(kmax))
    return kmin, kmax


def attend_tokens(q, K, V, tok, scale):
    q, K, V = f32(q), f32(K), f32(V)
    tok = np.ascontiguousarray(tok, dtype=np.int32)
    d = q.shape[-1]
    o = np.empty(d, np.float64)
    lse = np.empty(1, np.float64)
    _load().oracle_attend_tokens(ctypes.c_int(d), ctypes.c_float(scale), _f(q), _f(K), _f(V),
                                 ctypes.c_int(len(tok)), _i(tok), _d(o), _d(lse))
    return o, float(lse[0])


def merge(o1, l1, o2, l2):
    o1 = np.ascontiguousarray(o1, np.float64)
    o2 = np.ascontiguousarray(o2, np.float64)
    o = np.empty_like(o1)
    lse = np.empty(1, np.float64)
    _load().oracle_merge(ctypes.c_int(len(o1)), _d(o1), ctypes.c_double(l1), _d(o2),
                         ctypes.c_double(l2), _d(o), _d(lse))
    return o, float(lse[0])


def locality(sh: Shape, Qc, Qp):
    Qc, Qp = f32(Qc), f32(Qp)
    mse = np.empty((sh.S, sh.Hq, sh.B), np.float32)
    _load().oracle_locality(ctypes.byref(sh), _f(Qc), _f(Qp), _f(mse))
    return mse


def active(sh: Shape, mse):
    mse = f32(mse)
    out = np.empty((sh.S, sh.Hq, sh.A), np.int32)
    _load().oracle_active(ctypes.byref(sh), _f(mse), _i(out))
    return out


def bound_scores(q, kmin, kmax):
    q, kmin, kmax = f32(q), f32(kmin), f32(kmax)
    P, d = kmin.shape
    U = np.empty(P, np.float32)
    _load().oracle_bound_scores(ctypes.c_int(d), ctypes.c_int(P), _f(q), _f(kmin), _f(kmax), _f(U))
    return U


def topk_pages(U, k):
    U = f32(U)
    out = np.empty(k, np.int32)
    _load().oracle_topk_pages(ctypes.c_int(len(U)), ctypes.c_int(k), _f(U), _i(out))
    return out


def dense_prefix(sh: Shape, Q, K, V, Kb, Vb):
    """Cold-start pass.  Returns dict(o_p, l_p, out, lse)."""
    Q, K, V, Kb, Vb = map(f32, (Q, K, V, Kb, Vb))
    o_p = np.empty((sh.S, sh.Hq, sh.B, sh.d), np.float32)
    l_p = np.empty((sh.S, sh.Hq, sh.B), np.float32)
    out = np.empty_like(o_p)
    lse = np.empty_like(l_p)
    _load().oracle_dense_prefix(ctypes.byref(sh), _f(Q), _f(K), _f(V), _f(Kb), _f(Vb), _f(o_p),
                                _f(l_p), _f(out), _f(lse))
    return {"o_p": o_p, "l_p": l_p, "out": out, "lse": lse}


def dense_rows(sh: Shape, Q, K, V, rows):
    """Dense prefix attention of the listed flattened rows of ``[S][Hq][B]``."""
    Q, K, V = map(f32, (Q, K, V))
    rows = np.ascontiguousarray(rows, dtype=np.int32)
    o_p = np.empty((len(rows), sh.d), np.float32)
    l_p = np.empty(len(rows), np.float32)
    _load().oracle_dense_rows(ctypes.byref(sh), _f(Q), _f(K), _f(V), ctypes.c_int(len(rows)),
                              _i(rows), _f(o_p), _f(l_p))
    return o_p, l_p


def step(sh: Shape, Qc, Qp, K, V, kmin, kmax, Kb, Vb, o_p, l_p, want_bound=False):
    """One LoSA step.  ``o_p``/``l_p`` are the incoming cache; copies are
    updated and returned.  Returns dict(o_p, l_p, out, lse, active_idx,
    page_idx, union_count, mse[, bound])."""
    Qc, Qp, K, V, kmin, kmax, Kb, Vb = map(f32, (Qc, Qp, K, V, kmin, kmax, Kb, Vb))
    o_p = f32(o_p).copy()
    l_p = f32(l_p).copy()
    k = pages_per_row(sh)
    P = n_pages(sh)
    out = np.empty((sh.S, sh.Hq, sh.B, sh.d), np.float32)
    lse = np.empty((sh.S, sh.Hq, sh.B), np.float32)
    act = np.empty((sh.S, sh.Hq, sh.A), np.int32)
    pidx = np.empty((sh.S, sh.Hq, sh.A, k), np.int32)
    uc = np.empty((sh.S, sh.Hkv), np.int32)
    mse = np.empty((sh.S, sh.Hq, sh.B), np.float32)
    bound = np.empty((sh.S, sh.Hq, sh.A, P), np.float32) if want_bound else None
    _load().oracle_step(ctypes.byref(sh), _f(Qc), _f(Qp), _f(K), _f(V), _f(kmin), _f(kmax),
                        _f(Kb), _f(Vb), _f(o_p), _f(l_p), _f(out), _f(lse), _i(act), _i(pidx),
                        _i(uc), _f(mse), _opt(bound, _f))
    res = {"o_p": o_p, "l_p": l_p, "out": out, "lse": lse, "active_idx": act,
           "page_idx": pidx, "union_count": uc, "mse": mse}
    if want_bound:
        res["bound"] = bound
    return res


def step_forced(sh: Shape, Qc, K, V, Kb, Vb, active_idx, page_idx, o_p, l_p):
    """LoSA step with a given active set and page lists."""
    Qc, K, V, Kb, Vb = map(f32, (Qc, K, V, Kb, Vb))
    o_p = f32(o_p).copy()
    l_p = f32(l_p).copy()
    act = np.ascontiguousarray(active_idx, dtype=np.int32)
    pidx = np.ascontiguousarray(page_idx, dtype=np.int32)
    out = np.empty((sh.S, sh.Hq, sh.B, sh.d), np.float32)
    lse = np.empty((sh.S, sh.Hq, sh.B), np.float32)
    uc = np.empty((sh.S, sh.Hkv), np.int32)
    _load().oracle_step_forced(ctypes.byref(sh), _f(Qc), _f(K), _f(V), _f(Kb), _f(Vb), _i(act),
                               _i(pidx), _f(o_p), _f(l_p), _f(out), _f(lse), _i(uc))
    return {"o_p": o_p, "l_p": l_p, "out": out, "lse": lse, "union_count": uc}


def refresh_ref(sh: Shape, Qc, active_idx, q_ref):
    """Drift-safe locality: ``q_ref`` with the active rows' current queries
    moved in (a copy is returned)."""
    Qc = f32(Qc)
    q_ref = f32(q_ref).copy()
    act = np.ascontiguousarray(active_idx, dtype=np.int32)
    _load().oracle_refresh_ref(ctypes.byref(sh), _f(Qc), _i(act), _f(q_ref))
    return q_ref


def step_ref(sh: Shape, Qc, q_ref, K, V, kmin, kmax, Kb, Vb, o_p, l_p):
    """One drift-safe LoSA step: locality against the reference queries, then
    the reference refreshed for the recomputed rows.  Returns step()'s dict
    plus ``q_ref`` (the updated reference)."""
    res = step(sh, Qc, q_ref, K, V, kmin, kmax, Kb, Vb, o_p, l_p)
    res["q_ref"] = refresh_ref(sh, Qc, res["active_idx"], q_ref)
    return res

def append_block(K, V, Kb, Vb):
    """Prefix growth: the committed block's keys/values become prefix tokens
    L .. L+B-1 of every (sequence, KV head) -- a concatenation along the token
    axis of ``[S][Hkv][L][d]`` and ``[S][Hkv][B][d]``.  The grown prefix's
    page metadata is ``build_meta`` over the result."""
    return (np.concatenate([f32(K), f32(Kb)], axis=2), np.concatenate([f32(V), f32(Vb)], axis=2))

# ---------------------------------------------------------------------------
# Variable-length batches.  The pages define the step for one sequence; a
# batch whose sequences have different prefix lengths is read as what the
# definition gives for each sequence on its own (prefix length lens[s], its
# own pages P_s = ceil(lens[s] / ps) and k_s = min(budget / ps, P_s)), laid
# side by side.  Inputs are the batch's capacity-strided arrays
# ([S][Hkv][>= max lens][d]); tokens past a sequence's length are not read.
# Page lists are padded to the batch's k = min(budget / ps, P_max) with -1.
# ---------------------------------------------------------------------------
def seq_shape(sh: Shape, L: int) -> Shape:
    """The one-sequence shape of a sequence of prefix length ``L``."""
    return shape(1, sh.Hq, sh.Hkv, sh.d, int(L), sh.ps, sh.B, sh.A, sh.budget, sh.scale,
                 sh.flags)


def _seq_prefix(X, s, L):
    return f32(X[s:s + 1, :, :int(L)])


def build_meta_varlen(sh: Shape, lens, K):
    """Per-sequence page metadata: a list of (kmin, kmax), ``[1][Hkv][P_s][d]``."""
    return [build_meta(seq_shape(sh, L), _seq_prefix(K, s, L)) for s, L in enumerate(lens)]


def dense_prefix_varlen(sh: Shape, lens, Q, K, V, Kb, Vb):
    parts = [dense_prefix(seq_shape(sh, L), f32(Q[s:s + 1]), _seq_prefix(K, s, L),
                          _seq_prefix(V, s, L), f32(Kb[s:s + 1]), f32(Vb[s:s + 1]))
             for s, L in enumerate(lens)]
    return {key: np.concatenate([p[key] for p in parts]) for key in parts[0]}


def step_varlen(sh: Shape, lens, Qc, Qp, K, V, Kb, Vb, o_p, l_p):
    """One LoSA step of a variable-length batch (metadata built from K per
    sequence).  Returns step()'s dict, page_idx padded with -1."""
    k = pages_per_row(sh)
    parts = []
    for s, L in enumerate(lens):
        ssh = seq_shape(sh, L)
        Ks = _seq_prefix(K, s, L)
        kmin, kmax = build_meta(ssh, Ks)
        r = step(ssh, f32(Qc[s:s + 1]), f32(Qp[s:s + 1]), Ks, _seq_prefix(V, s, L), kmin, kmax,
                 f32(Kb[s:s + 1]), f32(Vb[s:s + 1]), f32(o_p[s:s + 1]), f32(l_p[s:s + 1]))
        pidx = np.full(r["page_idx"].shape[:-1] + (k,), -1, np.int32)
        pidx[..., :r["page_idx"].shape[-1]] = r["page_idx"]
        r["page_idx"] = pidx
        parts.append(r)
    return {key: np.concatenate([p[key] for p in parts]) for key in parts[0]}


def append_block_varlen(lens, K, V, Kb, Vb):
    """Each sequence's block appended at its own length: a list of the grown
    ``(K_s, V_s)``, ``[1][Hkv][lens[s] + B][d]``."""
    return [append_block(_seq_prefix(K, s, L), _seq_prefix(V, s, L), f32(Kb[s:s + 1]),
                         f32(Vb[s:s + 1])) for s, L in enumerate(lens)]
