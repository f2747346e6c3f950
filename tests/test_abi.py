"""The C-ABI library without a GPU: it builds, loads, exports every symbol the
header declares, and its host-side validation returns the documented codes
before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

from sparse_long_context_mse_b200 import api, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "losa.h")


@pytest.fixture(scope="module")
def L():
    build.build()
    return api.lib()


def header_functions():
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(losa_[a-z_]+)\s*\(", txt)))


def test_exports_every_declared_symbol(L):
    declared = header_functions()
    assert set(declared) == set(api.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name
    nm = subprocess.run(["nm", "-D", "--defined-only", api.LIB_PATH], capture_output=True,
                        text=True).stdout
    for name in declared:
        assert re.search(rf"\bT {name}\b", nm), f"{name} not exported"


def test_library_is_sm100a_only():
    # the build targets sm_100a only (no other SASS, no PTX for JIT)
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)


def S(**kw):
    base = dict(num_seqs=1, n_q_heads=32, n_kv_heads=8, head_dim=128, prefix_len=65536,
                page_size=16, block_size=16, n_active=4, token_budget=128, dtype="bf16")
    base.update(kw)
    return api.make_shape(**base)


@pytest.fixture
def no_device():
    """Validation tests that pass fake addresses: a call that wrongly passed
    validation would launch on them, so they run only without a GPU."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("fake device addresses: CPU-only validation test")


def test_status_strings(L):
    for code in range(6):
        assert api.status_string(code)
    assert api.status_string(99) == "unknown status"


def test_sizes(L):
    sh = S()
    P = 4096

    def norms(Pc):  # the page-norm rows: float2 per page, rows padded to 8 pages
        return 8 * ((Pc + 7) // 8 * 8) * 8

    assert api.page_meta_size(sh) == 8 * P * 2 * 128 * 2 + norms(P)
    assert api.page_meta_size(S(dtype="f32")) == 8 * P * 2 * 128 * 4 + norms(P)
    assert api.page_meta_size(S(prefix_len=65537)) == 8 * (P + 1) * 2 * 128 * 2 + norms(P + 1)
    for which in (api.LOSA_WS_DENSE, api.LOSA_WS_STEP):
        n = api.workspace_size(sh, which)
        assert n > 0 and n % 256 == 0
    assert api.workspace_size(sh, 7) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(n_q_heads=30), api.LOSA_ERR_INVALID_ARG),          # Hq % Hkv != 0
    (dict(n_active=17), api.LOSA_ERR_INVALID_ARG),           # |A| > B
    (dict(n_active=-1), api.LOSA_ERR_INVALID_ARG),
    (dict(prefix_len=0), api.LOSA_ERR_INVALID_ARG),
    (dict(token_budget=8), api.LOSA_ERR_INVALID_ARG),         # k = 0 with |A| > 0
    (dict(scale=-1.0), api.LOSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), api.LOSA_ERR_INVALID_ARG),
    (dict(head_dim=64), api.LOSA_ERR_UNSUPPORTED),
    (dict(page_size=32), api.LOSA_ERR_UNSUPPORTED),
    (dict(dtype=7), api.LOSA_ERR_UNSUPPORTED),
    (dict(block_size=64, n_active=4), api.LOSA_ERR_UNSUPPORTED),   # B > 32
    (dict(n_q_heads=64, n_kv_heads=2, block_size=8), api.LOSA_ERR_UNSUPPORTED),  # G*B > 128
    (dict(token_budget=16 * 65), api.LOSA_ERR_UNSUPPORTED),  # 64 < k < P
])
def test_shape_validation(L, kw, code):
    if kw.get("dtype") == 7:
        sh = S()
        sh.dtype = 7
    else:
        sh = S(**kw)
    assert api.workspace_size(sh, api.LOSA_WS_STEP) == 0
    fake = ctypes.c_void_p(1 << 20)
    rc = L.losa_step(ctypes.byref(sh), *([fake] * 10), None, None, None, None, fake,
                     1 << 40, None)
    assert rc == code
    rc = L.losa_build_page_meta(ctypes.byref(sh), fake, ctypes.c_void_p(1 << 30), None)
    assert rc == code


def test_legal_edge_shapes_size(L):
    # |A| = 0 with a zero budget, and k == P beyond 64 (every page), are legal
    assert api.workspace_size(S(n_active=0, token_budget=0), api.LOSA_WS_STEP) > 0
    assert api.workspace_size(S(prefix_len=4096, token_budget=4096), api.LOSA_WS_STEP) > 0
    assert api.workspace_size(S(n_q_heads=8, n_kv_heads=1, block_size=16, n_active=16,
                                prefix_len=3000), api.LOSA_WS_STEP) > 0
    # 128 active rows per KV head over a 64K prefix (smaller scan chunks)
    assert api.workspace_size(S(n_q_heads=8, n_kv_heads=1, block_size=16, n_active=16),
                              api.LOSA_WS_STEP) > 0


def _step_args(ptrs):
    return [ctypes.c_void_p(p) if p is not None else None for p in ptrs]


# fake device addresses 64 GiB apart: no two buffers of a call overlap
FAR = [(i + 1) << 36 for i in range(16)]


def test_pointer_validation(L, no_device):
    sh = S()
    ws_n = api.workspace_size(sh, api.LOSA_WS_STEP)
    base = FAR[:10] + [None, None, None, None, FAR[14]]

    def call(ptrs, ws_bytes=ws_n):
        return L.losa_step(ctypes.byref(sh), *_step_args(ptrs), ws_bytes, None)

    for i in range(10):  # each required pointer: null, then misaligned
        p = list(base)
        p[i] = None
        assert call(p) == api.LOSA_ERR_INVALID_ARG
        p[i] = base[i] + 8
        assert call(p) == api.LOSA_ERR_INVALID_ARG
    p = list(base)
    p[14] = base[14] + 128               # workspace not 256-byte aligned
    assert call(p) == api.LOSA_ERR_INVALID_ARG
    assert call(base, ws_n - 1) == api.LOSA_ERR_INVALID_ARG   # workspace too small
    p = list(base)
    p[11] = 0x900004                     # optional output misaligned
    assert call(p) == api.LOSA_ERR_INVALID_ARG
    assert L.losa_step(None, *_step_args(base), ws_n, None) == api.LOSA_ERR_INVALID_ARG


# (written buffer, other buffer) index pairs of losa_step's pointer list:
# 0 q_cur 1 q_prev 2 k_prefix 3 v_prefix 4 page_meta 5 k_blk 6 v_blk 7 o_p
# 8 l_p 9 out 10 out_lse 11 active_idx 12 page_idx 13 union_count 14 workspace
STEP_ALIASES = [(9, 0), (9, 2), (9, 3), (9, 4), (9, 5), (9, 6), (9, 7), (9, 14), (10, 1),
                (10, 8), (10, 14), (7, 14), (8, 14), (7, 2), (8, 4), (11, 12), (12, 14),
                (13, 3), (11, 7)]


@pytest.mark.parametrize("w,o", STEP_ALIASES)
def test_step_refuses_written_aliases(L, w, o, no_device):
    # a written buffer overlapping any other buffer of the call is refused
    # before anything is launched; the address sits inside the other buffer
    # (with fake addresses a call that passed validation would launch, so the
    # test only runs where there is no device to launch on)
    sh = S()
    ws_n = api.workspace_size(sh, api.LOSA_WS_STEP)
    p = list(FAR[:15])
    p[w] = p[o] + 16             # 16 bytes into the other buffer (every one is larger)
    rc = L.losa_step(ctypes.byref(sh), *_step_args(p), ws_n, None)
    assert rc == api.LOSA_ERR_INVALID_ARG


def test_step_flags_validation(L, no_device):
    # the union variant is a legal step shape; an unknown bit is refused
    # before anything is launched
    assert api.workspace_size(S(flags=api.LOSA_STEP_ATTEND_UNION), api.LOSA_WS_STEP) > 0
    bad = S(flags=2)
    assert api.workspace_size(bad, api.LOSA_WS_STEP) == 0
    fake = ctypes.c_void_p(1 << 20)
    assert L.losa_step(ctypes.byref(bad), *([fake] * 10), None, None, None, None, fake,
                       1 << 40, None) == api.LOSA_ERR_INVALID_ARG


def test_step_ref_pointer_validation(L, no_device):
    # losa_step_ref rewrites q_ref: null, or aliasing any output or q_cur, is
    # refused before anything is launched
    sh = S()
    ws_n = api.workspace_size(sh, api.LOSA_WS_STEP)
    base = FAR[:10] + [None, None, None, None, FAR[14]]

    def call(ptrs):
        return L.losa_step_ref(ctypes.byref(sh), *_step_args(ptrs), ws_n, None)

    for i, other in ((1, None), (1, 0), (1, 7), (1, 8), (1, 9)):
        p = list(base)
        p[i] = None if other is None else base[other]
        assert call(p) == api.LOSA_ERR_INVALID_ARG, other
    p = list(base)
    p[10] = base[1]                      # out_lse aliases q_ref
    assert call(p) == api.LOSA_ERR_INVALID_ARG


def test_prefix_capacity_validation(L, no_device):
    # a capacity below the prefix length is refused; a larger one grows the
    # metadata to ceil(capacity / ps) records per (s, g)
    assert api.workspace_size(S(prefix_capacity=65535), api.LOSA_WS_STEP) == 0
    assert api.page_meta_size(S(prefix_capacity=65536 + 33)) == (8 * (4096 + 3) * 2 * 128 * 2 +
                                                                 8 * 4104 * 8)
    # appending a block needs room for B more tokens: refused before any launch
    fake = [ctypes.c_void_p((i + 1) << 36) for i in range(5)]  # far apart: no overlaps
    assert L.losa_append_block(ctypes.byref(S(prefix_capacity=65536 + 15)), *fake,
                               None) == api.LOSA_ERR_INVALID_ARG
    assert L.losa_append_block(ctypes.byref(S()), *fake, None) == api.LOSA_ERR_INVALID_ARG
    fake[2] = fake[0]                    # k_prefix aliases k_blk
    assert L.losa_append_block(ctypes.byref(S(prefix_capacity=65536 + 16)), *fake,
                               None) == api.LOSA_ERR_INVALID_ARG


def test_prefix_lens_validation(L):
    # the per-sequence length array is a device pointer read by the kernels:
    # the host checks only its alignment, and the sizes follow prefix_len
    # (the largest length)
    sh = S()
    sh.prefix_lens = 0x100002
    assert api.workspace_size(sh, api.LOSA_WS_STEP) == 0
    assert api.page_meta_size(sh) == 0
    sh.prefix_lens = 0x100004
    for which in (api.LOSA_WS_STEP, api.LOSA_WS_DENSE):
        assert api.workspace_size(sh, which) == api.workspace_size(S(), which) > 0
    assert api.page_meta_size(sh) == api.page_meta_size(S())
    assert ctypes.sizeof(api.Shape) == 13 * 4 + 4 + 8  # 8-byte aligned pointer last
    import copy
    c = copy.copy(sh)
    c.prefix_len = 7
    assert c.prefix_lens == sh.prefix_lens and sh.prefix_len == 65536
    import torch
    with pytest.raises(ValueError):  # a host tensor is refused by the binding
        api.make_shape(2, 8, 2, 128, 100, 16, 16, 4, 64,
                       prefix_lens=torch.tensor([100, 50], dtype=torch.int32))


def test_prefix_lens_on_another_device_is_refused(L):
    # the binding refuses, before any launch, a length array that lives on
    # another GPU than the call's tensors (no GPU is needed to check this)
    import types
    import torch
    sh = S()
    sh.prefix_lens = 0x100000
    sh._prefix_lens = types.SimpleNamespace(device=torch.device("cuda", 1))
    t = types.SimpleNamespace(device=torch.device("cuda", 0))
    with pytest.raises(ValueError):
        api._call_device(sh, t)
    sh._prefix_lens = types.SimpleNamespace(device=torch.device("cuda", 0))
    assert api._call_device(sh, t) == torch.device("cuda", 0)
    assert api._call_device(S(), t) == torch.device("cuda", 0)


def test_dense_pointer_validation(L, no_device):
    sh = S()
    ws_n = api.workspace_size(sh, api.LOSA_WS_DENSE)
    base = FAR[:9] + [FAR[14]]
    for i in range(8):
        p = list(base)
        p[i] = None
        rc = L.losa_dense_prefix(ctypes.byref(sh), *_step_args(p), ws_n, None)
        assert rc == api.LOSA_ERR_INVALID_ARG
    rc = L.losa_dense_prefix(ctypes.byref(sh), *_step_args(base), ws_n - 256, None)
    assert rc == api.LOSA_ERR_INVALID_ARG
    # 0 q 1 k_prefix 2 v_prefix 3 k_blk 4 v_blk 5 o_p 6 l_p 7 out 8 out_lse 9 workspace
    for w, o in ((7, 0), (7, 1), (7, 5), (8, 9), (5, 2), (6, 3), (5, 9), (8, 6)):
        p = list(base)
        p[w] = p[o] + 16
        rc = L.losa_dense_prefix(ctypes.byref(sh), *_step_args(p), ws_n, None)
        assert rc == api.LOSA_ERR_INVALID_ARG, (w, o)


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(api, "_lib", None)
    monkeypatch.setattr(api, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError, match="missing"):
        api.lib()


def test_product_library_has_no_phase_trace(L):
    # the per-phase timestamps exist only in the separate tracing build
    assert not hasattr(L, "losa_phase_read")
    assert not hasattr(L, "losa_phase_clear")
