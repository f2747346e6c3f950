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
        for key in ("active_idx", "page_idx", "union_count"):
            assert torch.equal(got[key], ref[key]), (call, key)
        for key in ("out", "lse"):
            e = maxabs(got[key].cpu().numpy(), ref[key].cpu().numpy())
            assert e <= TOL, (call, key, e)
        assert maxabs(o_p.cpu().numpy(), ref_o.cpu().numpy()) <= TOL, call
        assert maxabs(l_p.cpu().numpy(), ref_l.cpu().numpy()) <= TOL, call


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # sixteen 64K sequences with every block token active and a 1024-token
    # budget need more step workspace than the fixed array holds: refused
    # before anything is launched (the fake pointers are never dereferenced)
    sh = api.make_shape(16, 32, 8, 128, 65536, 16, 16, 16, 1024)
    assert api.workspace_size(sh, api.LOSA_WS_STEP) > api.NOALLOC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)
    rc = api.lib().losa_step_noalloc(ctypes.byref(sh), *([fake] * 10), None, None, None, None,
                                     None)
    assert rc == api.LOSA_ERR_UNSUPPORTED
    bad = api.make_shape(1, 30, 8, 128, 4096, 16, 16, 4, 128)
    assert api.lib().losa_step_noalloc(ctypes.byref(bad), *([fake] * 10), None, None, None,
                                       None, None) == api.LOSA_ERR_INVALID_ARG
    assert np.isfinite(TOL)
