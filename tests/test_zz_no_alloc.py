"""losa_step_noalloc: the step entry point for callers that cannot allocate
device memory (it runs on a fixed scratch array owned by the library instead
of a caller workspace).  Its results must match losa_step with a caller
workspace, call after call.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

from losa_testutil import DEV, TOL, Case, gpu_dense, gpu_meta, maxabs
from sparse_long_context_mse_b200 import api, synth

pytestmark = pytest.mark.gpu


def _outputs(sh):
    import torch
    rows = (sh.num_seqs, sh.n_q_heads, sh.block_size)
    A, k = sh.n_active, sh.pages_per_row
    return {"out": torch.empty(*rows, sh.head_dim, device=DEV),
            "lse": torch.empty(*rows, device=DEV),
            "active_idx": torch.empty(sh.num_seqs, sh.n_q_heads, A, dtype=torch.int32, device=DEV),
            "page_idx": torch.empty(sh.num_seqs, sh.n_q_heads, A, k, dtype=torch.int32,
                                    device=DEV),
            "union_count": torch.empty(sh.num_seqs, sh.n_kv_heads, dtype=torch.int32,
                                       device=DEV)}


def test_noalloc_matches_workspace_step_on_two_calls():
    import torch
    c = Case(synth.workload(synth.GQA16K))
    sh = c.sh
    assert api.workspace_size(sh, api.LOSA_WS_STEP) <= api.NOALLOC_SCRATCH_BYTES
    meta = gpu_meta(sh, c.K)
    cache = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])

    # the existing entry point, with a workspace the caller allocated
    ref = _outputs(sh)
    ref_o, ref_l = cache["o_p"].clone(), cache["l_p"].clone()
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, DEV)
    api.step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], ref_o, ref_l, ref["out"],
             ref["lse"], ws, ref["active_idx"], ref["page_idx"], ref["union_count"])

    for call in range(2):
        got = _outputs(sh)
        o_p, l_p = cache["o_p"].clone(), cache["l_p"].clone()
        api.step_noalloc(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], o_p, l_p,
                         got["out"], got["lse"], got["active_idx"], got["page_idx"],
                         got["union_count"])
        torch.cuda.synchronize()
        assert api.noalloc_read_status() == api.LOSA_OK, call
        for key in ("active_idx", "page_idx", "union_count"):
            assert torch.equal(got[key], ref[key]), (call, key)
        for key in ("out", "lse"):
            e = maxabs(got[key].cpu().numpy(), ref[key].cpu().numpy())
            assert e <= TOL, (call, key, e)
        assert maxabs(o_p.cpu().numpy(), ref_o.cpu().numpy()) <= TOL, call
        assert maxabs(l_p.cpu().numpy(), ref_l.cpu().numpy()) <= TOL, call


def test_noalloc_fits_every_workload_and_refuses_bad_shapes():
    # the step keeps its working state in shared memory; its workspace (and
    # so the fixed array's used part) is the status word, for every workload
    for w in (synth.TINY, synth.GQA16K, synth.GQA64K, synth.BATCH8, synth.STACK36):
        sh = api.shape_of(synth.workload(w).for_layer(0))
        assert 0 < api.workspace_size(sh, api.LOSA_WS_STEP) <= api.NOALLOC_SCRATCH_BYTES, w
    # an invalid shape is refused before anything is launched (the fake
    # pointers are never dereferenced)
    fake = ctypes.c_void_p(1 << 20)
    bad = api.make_shape(1, 30, 8, 128, 4096, 16, 16, 4, 128)
    assert api.lib().losa_step_noalloc(ctypes.byref(bad), *([fake] * 10), None, None, None,
                                       None, None) == api.LOSA_ERR_INVALID_ARG
    assert np.isfinite(TOL)


def _compare_with_workspace_step(sh, c, meta, cache):
    """One noalloc call against losa_step on a freshly zeroed workspace."""
    import torch
    ref, got = _outputs(sh), _outputs(sh)
    ref_o, ref_l = cache["o_p"].clone(), cache["l_p"].clone()
    o_p, l_p = cache["o_p"].clone(), cache["l_p"].clone()
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, DEV)
    api.step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], ref_o, ref_l, ref["out"],
             ref["lse"], ws, ref["active_idx"], ref["page_idx"], ref["union_count"])
    api.step_noalloc(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], o_p, l_p,
                     got["out"], got["lse"], got["active_idx"], got["page_idx"],
                     got["union_count"])
    torch.cuda.synchronize()
    assert api.read_device_status(ws) == api.LOSA_OK
    assert api.noalloc_read_status() == api.LOSA_OK
    for key in ("active_idx", "page_idx", "union_count"):
        assert torch.equal(got[key], ref[key]), key
    for key in ("out", "lse"):
        assert maxabs(got[key].cpu().numpy(), ref[key].cpu().numpy()) <= TOL, key
    assert maxabs(o_p.cpu().numpy(), ref_o.cpu().numpy()) <= TOL
    assert maxabs(l_p.cpu().numpy(), ref_l.cpu().numpy()) <= TOL


def test_noalloc_shape_changes_leave_no_trace():
    """Calls of different shapes in a row share the scratch array: a uniform
    batch, then a variable-length one, then a smaller budget and more active
    tokens; each must equal losa_step on a fresh workspace."""
    import torch
    from losa_testutil import random_case
    c = random_case(3, 8, 2, 700, 16, 4, 96, "bf16", seed=5)
    shapes = []
    shapes.append(c.sh)
    lens = torch.tensor([700, 33, 410], dtype=torch.int32, device=DEV)
    shapes.append(api.make_shape(3, 8, 2, 128, 700, 16, 16, 4, 96, "bf16", scale=c.sh.scale,
                                 prefix_lens=lens))
    shapes.append(api.make_shape(3, 8, 2, 128, 700, 16, 16, 7, 32, "bf16", scale=c.sh.scale))
    for sh in shapes:
        meta = gpu_meta(sh, c.K)
        cache = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
        _compare_with_workspace_step(sh, c, meta, cache)


def test_noalloc_status_reports_and_clears_bounds():
    """An out-of-range per-sequence length is clamped and reported as
    LOSA_ERR_DEVICE_BOUNDS through the noalloc status; reading clears it."""
    import torch
    from losa_testutil import random_case
    c = random_case(2, 8, 2, 300, 16, 4, 64, "bf16", seed=6)
    sh0 = c.sh
    meta = gpu_meta(sh0, c.K)
    cache = gpu_dense(sh0, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    lens = torch.tensor([300, 301], dtype=torch.int32, device=DEV)  # 301 > prefix_len
    sh = api.make_shape(2, 8, 2, 128, 300, 16, 16, 4, 64, "bf16", scale=sh0.scale,
                        prefix_lens=lens)
    got = _outputs(sh)
    o_p, l_p = cache["o_p"].clone(), cache["l_p"].clone()
    assert api.noalloc_read_status() == api.LOSA_OK
    api.step_noalloc(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], o_p, l_p,
                     got["out"], got["lse"], got["active_idx"], got["page_idx"],
                     got["union_count"])
    assert api.noalloc_read_status() == api.LOSA_ERR_DEVICE_BOUNDS
    assert api.noalloc_read_status() == api.LOSA_OK
    # the clamped call equals the in-range one
    ok = _outputs(sh0)
    o2, l2 = cache["o_p"].clone(), cache["l_p"].clone()
    api.step_noalloc(sh0, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], o2, l2,
                     ok["out"], ok["lse"], ok["active_idx"], ok["page_idx"], ok["union_count"])
    assert api.noalloc_read_status() == api.LOSA_OK
    for key in ("active_idx", "page_idx", "union_count"):
        assert torch.equal(got[key], ok[key]), key
