"""Thin Python binding of the LoSA C ABI (``include/losa.h``).

Argument marshalling only: every function checks dtype, shape, device and
contiguity of the torch tensors it is given, then passes raw device pointers
and the current CUDA stream to ``liblosa.so``.  All compute happens in the
library's kernels.  There is no fallback: if the library is missing or a
call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "liblosa.so")

LOSA_OK = 0
LOSA_ERR_INVALID_ARG = 1
LOSA_ERR_UNSUPPORTED = 2
LOSA_ERR_CUDA = 3
LOSA_ERR_DEVICE_TIMEOUT = 4
LOSA_ERR_DEVICE_BOUNDS = 5
LOSA_F32 = 0
LOSA_BF16 = 1
LOSA_STEP_ATTEND_UNION = 1  # losa_shape.flags: active rows attend to the group's whole union
LOSA_WS_DENSE = 0
LOSA_WS_STEP = 1

#: every symbol ``include/losa.h`` declares
EXPORTS = ("losa_page_meta_size", "losa_workspace_size", "losa_build_page_meta",
           "losa_dense_prefix", "losa_step", "losa_step_ref", "losa_step_noalloc",
           "losa_append_block",
           "losa_read_device_status", "losa_noalloc_read_status",
           "losa_status_string", "losa_last_error")

#: size of the library-owned scratch behind ``losa_step_noalloc``
NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


class LosaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"losa status {code}: {msg}")
        self.code = code


class Shape(ctypes.Structure):
    """``losa_shape``."""
    _fields_ = [("num_seqs", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("prefix_len", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("n_active", ctypes.c_int32),
                ("token_budget", ctypes.c_int32), ("scale", ctypes.c_float),
                ("dtype", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("prefix_capacity", ctypes.c_int32), ("prefix_lens", ctypes.c_void_p)]

    def __copy__(self):
        """A field-by-field copy (ctypes cannot pickle a structure that holds a
        pointer); it shares the per-sequence length array."""
        sh = Shape(*(getattr(self, f) for f, _ in self._fields_))
        sh._prefix_lens = getattr(self, "_prefix_lens", None)
        return sh

    # derived sizes (same rules as the library's validation)
    @property
    def group(self):
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_pages(self):
        return (self.prefix_len + self.page_size - 1) // self.page_size

    @property
    def capacity(self):
        """Tokens per (sequence, KV head) in the prefix buffers."""
        return self.prefix_capacity if self.prefix_capacity > 0 else self.prefix_len

    @property
    def pages_per_row(self):
        return min(self.token_budget // self.page_size, self.n_pages)

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == LOSA_BF16 else torch.float32


def make_shape(num_seqs, n_q_heads, n_kv_heads, head_dim, prefix_len, page_size, block_size,
               n_active, token_budget, dtype="bf16", scale: Optional[float] = None,
               flags: int = 0, prefix_capacity: int = 0, prefix_lens=None) -> Shape:
    """``prefix_lens``: None, or an int32 device tensor of ``num_seqs`` per-sequence
    prefix lengths (a variable-length batch; ``prefix_len`` is then the largest).
    The shape keeps a reference to it and passes its address: the library reads
    its current contents at every call."""
    dt = {"bf16": LOSA_BF16, "f32": LOSA_F32, LOSA_BF16: LOSA_BF16, LOSA_F32: LOSA_F32}[dtype]
    sc = float(scale) if scale is not None else 0.0
    lens_ptr = None
    if prefix_lens is not None:
        if (prefix_lens.dtype != torch.int32 or not prefix_lens.is_contiguous()
                or prefix_lens.numel() != num_seqs or prefix_lens.device.type != "cuda"):
            raise ValueError("prefix_lens: a contiguous int32 CUDA tensor of num_seqs entries")
        lens_ptr = prefix_lens.data_ptr()
    sh = Shape(num_seqs, n_q_heads, n_kv_heads, head_dim, prefix_len, page_size, block_size,
               n_active, token_budget, sc, dt, flags, prefix_capacity, lens_ptr)
    sh._prefix_lens = prefix_lens  # keeps the array alive as long as the shape
    return sh


def shape_of(cfg, scale: Optional[float] = None, flags: int = 0) -> Shape:
    """Shape of a :class:`synth.LosaConfig` (duck-typed)."""
    return make_shape(cfg.num_seqs, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim, cfg.prefix_len,
                      cfg.page_size, cfg.block_size, cfg.n_active, cfg.token_budget, cfg.dtype,
                      scale, flags)


_lib = None


def lib():
    """The loaded ``liblosa.so`` (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m sparse_long_context_mse_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        sp = ctypes.POINTER(Shape)
        L.losa_page_meta_size.argtypes = [sp]
        L.losa_page_meta_size.restype = sz
        L.losa_workspace_size.argtypes = [sp, i32]
        L.losa_workspace_size.restype = sz
        L.losa_build_page_meta.argtypes = [sp, vp, vp, vp]
        L.losa_build_page_meta.restype = i32
        L.losa_dense_prefix.argtypes = [sp] + [vp] * 9 + [vp, sz, vp]
        L.losa_dense_prefix.restype = i32
        L.losa_step.argtypes = [sp] + [vp] * 14 + [vp, sz, vp]
        L.losa_step.restype = i32
        L.losa_append_block.argtypes = [sp] + [vp] * 6
        L.losa_append_block.restype = i32
        L.losa_step_ref.argtypes = [sp] + [vp] * 14 + [vp, sz, vp]
        L.losa_step_ref.restype = i32
        L.losa_step_noalloc.argtypes = [sp] + [vp] * 14 + [vp]
        L.losa_step_noalloc.restype = i32
        L.losa_noalloc_read_status.argtypes = [vp]
        L.losa_noalloc_read_status.restype = i32
        L.losa_read_device_status.argtypes = [vp, vp]
        L.losa_read_device_status.restype = i32
        L.losa_status_string.argtypes = [i32]
        L.losa_status_string.restype = ctypes.c_char_p
        L.losa_last_error.argtypes = []
        L.losa_last_error.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().losa_status_string(code).decode()


def _check(code: int):
    if code != LOSA_OK:
        msg = status_string(code)
        if code == LOSA_ERR_CUDA:
            msg += " (" + lib().losa_last_error().decode() + ")"
        raise LosaError(code, msg)


def page_meta_size(sh: Shape) -> int:
    return lib().losa_page_meta_size(ctypes.byref(sh))


def workspace_size(sh: Shape, which: int) -> int:
    return lib().losa_workspace_size(ctypes.byref(sh), which)


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: Optional[torch.Tensor], shape, dtype, name, device):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _device_of(t: torch.Tensor):
    if t.device.type != "cuda":
        raise ValueError("tensors must live on a CUDA device")
    return t.device


def _call_device(sh: Shape, t: torch.Tensor):
    """The call's device (its first tensor's).  The shape's per-sequence length
    array, when it has one, must live there too: the kernels dereference it."""
    dev = _device_of(t)
    lens = getattr(sh, "_prefix_lens", None)
    if sh.prefix_lens and lens is not None and lens.device != dev:
        raise ValueError(f"prefix_lens lives on {lens.device}, the call's tensors on {dev}")
    return dev


def alloc_page_meta(sh: Shape, device) -> torch.Tensor:
    n = page_meta_size(sh)
    if n == 0:
        _check(LOSA_ERR_INVALID_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device)


def alloc_workspace(sh: Shape, which: int, device) -> torch.Tensor:
    n = workspace_size(sh, which)
    if n == 0:
        _check(LOSA_ERR_INVALID_ARG)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def build_page_meta(sh: Shape, k_prefix: torch.Tensor, page_meta: torch.Tensor, stream=None):
    dev = _call_device(sh, k_prefix)
    kv = (sh.num_seqs, sh.n_kv_heads, sh.capacity, sh.head_dim)
    a = _ptr(k_prefix, kv, sh.torch_dtype, "k_prefix", dev)
    b = _ptr(page_meta, (page_meta_size(sh),), torch.uint8, "page_meta", dev)
    _check(lib().losa_build_page_meta(ctypes.byref(sh), a, b, _stream(stream)))


def append_block(sh: Shape, k_blk, v_blk, k_prefix, v_prefix, page_meta, stream=None):
    """``losa_append_block``: commit a finished block to the prefix (tokens
    L .. L+B-1 of every (sequence, KV head)) and rebuild the page records it
    touches.  ``sh`` is the shape before the append; the prefix buffers need
    room for L + B tokens (``prefix_capacity``)."""
    dev = _call_device(sh, k_blk)
    kv = (sh.num_seqs, sh.n_kv_heads, sh.capacity, sh.head_dim)
    kb = (sh.num_seqs, sh.n_kv_heads, sh.block_size, sh.head_dim)
    args = [_ptr(k_blk, kb, sh.torch_dtype, "k_blk", dev), _ptr(v_blk, kb, sh.torch_dtype, "v_blk", dev),
            _ptr(k_prefix, kv, sh.torch_dtype, "k_prefix", dev),
            _ptr(v_prefix, kv, sh.torch_dtype, "v_prefix", dev),
            _ptr(page_meta, (page_meta_size(sh),), torch.uint8, "page_meta", dev)]
    _check(lib().losa_append_block(ctypes.byref(sh), *args, _stream(stream)))


def dense_prefix(sh: Shape, q, k_prefix, v_prefix, k_blk, v_blk, o_p, l_p, out, out_lse,
                 workspace, stream=None):
    dev = _call_device(sh, q)
    dt = sh.torch_dtype
    qs = (sh.num_seqs, sh.n_q_heads, sh.block_size, sh.head_dim)
    kv = (sh.num_seqs, sh.n_kv_heads, sh.capacity, sh.head_dim)
    kb = (sh.num_seqs, sh.n_kv_heads, sh.block_size, sh.head_dim)
    rs = qs[:3]
    args = [_ptr(q, qs, dt, "q", dev), _ptr(k_prefix, kv, dt, "k_prefix", dev),
            _ptr(v_prefix, kv, dt, "v_prefix", dev), _ptr(k_blk, kb, dt, "k_blk", dev),
            _ptr(v_blk, kb, dt, "v_blk", dev), _ptr(o_p, qs, torch.float32, "o_p", dev),
            _ptr(l_p, rs, torch.float32, "l_p", dev), _ptr(out, qs, torch.float32, "out", dev),
            _ptr(out_lse, rs, torch.float32, "out_lse", dev),
            _ptr(workspace, None, torch.uint8, "workspace", dev)]
    _check(lib().losa_dense_prefix(ctypes.byref(sh), *args, workspace.numel(), _stream(stream)))


def step(sh: Shape, q_cur, q_prev, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p, l_p, out,
         out_lse, workspace, active_idx=None, page_idx=None, union_count=None, stream=None):
    _step_call("losa_step", sh, q_cur, q_prev, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p,
               l_p, out, out_lse, workspace, active_idx, page_idx, union_count, stream)


def step_ref(sh: Shape, q_cur, q_ref, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p, l_p,
             out, out_lse, workspace, active_idx=None, page_idx=None, union_count=None,
             stream=None):
    """``losa_step_ref``: drift-safe locality.  ``q_ref`` holds each row's
    reference query (the one its cached o_p/L_p came from); the active rows'
    entries are overwritten with ``q_cur``."""
    _step_call("losa_step_ref", sh, q_cur, q_ref, k_prefix, v_prefix, page_meta, k_blk, v_blk,
               o_p, l_p, out, out_lse, workspace, active_idx, page_idx, union_count, stream)


def _step_call(fn, sh: Shape, q_cur, q_prev, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p,
               l_p, out, out_lse, workspace, active_idx, page_idx, union_count, stream):
    dev = _call_device(sh, q_cur)
    dt = sh.torch_dtype
    qs = (sh.num_seqs, sh.n_q_heads, sh.block_size, sh.head_dim)
    kv = (sh.num_seqs, sh.n_kv_heads, sh.capacity, sh.head_dim)
    kb = (sh.num_seqs, sh.n_kv_heads, sh.block_size, sh.head_dim)
    rs = qs[:3]
    A, k = sh.n_active, sh.pages_per_row
    args = [_ptr(q_cur, qs, dt, "q_cur", dev), _ptr(q_prev, qs, dt, "q_prev", dev),
            _ptr(k_prefix, kv, dt, "k_prefix", dev), _ptr(v_prefix, kv, dt, "v_prefix", dev),
            _ptr(page_meta, (page_meta_size(sh),), torch.uint8, "page_meta", dev),
            _ptr(k_blk, kb, dt, "k_blk", dev), _ptr(v_blk, kb, dt, "v_blk", dev),
            _ptr(o_p, qs, torch.float32, "o_p", dev), _ptr(l_p, rs, torch.float32, "l_p", dev),
            _ptr(out, qs, torch.float32, "out", dev),
            _ptr(out_lse, rs, torch.float32, "out_lse", dev),
            _ptr(active_idx, (sh.num_seqs, sh.n_q_heads, A), torch.int32, "active_idx", dev),
            _ptr(page_idx, (sh.num_seqs, sh.n_q_heads, A, k), torch.int32, "page_idx", dev),
            _ptr(union_count, (sh.num_seqs, sh.n_kv_heads), torch.int32, "union_count", dev),
            _ptr(workspace, None, torch.uint8, "workspace", dev)]
    _check(getattr(lib(), fn)(ctypes.byref(sh), *args, workspace.numel(), _stream(stream)))


def step_noalloc(sh: Shape, q_cur, q_prev, k_prefix, v_prefix, page_meta, k_blk, v_blk, o_p,
                 l_p, out, out_lse, active_idx=None, page_idx=None, union_count=None,
                 stream=None):
    """``losa_step_noalloc``: one step without a caller workspace, for callers
    that cannot allocate device memory (the library's own fixed scratch array
    is used; shapes needing more than ``NOALLOC_SCRATCH_BYTES`` are refused).
    Calls that may overlap on the GPU race on that array."""
    dev = _call_device(sh, q_cur)
    dt = sh.torch_dtype
    qs = (sh.num_seqs, sh.n_q_heads, sh.block_size, sh.head_dim)
    kv = (sh.num_seqs, sh.n_kv_heads, sh.capacity, sh.head_dim)
    kb = (sh.num_seqs, sh.n_kv_heads, sh.block_size, sh.head_dim)
    rs = qs[:3]
    A, k = sh.n_active, sh.pages_per_row
    args = [_ptr(q_cur, qs, dt, "q_cur", dev), _ptr(q_prev, qs, dt, "q_prev", dev),
            _ptr(k_prefix, kv, dt, "k_prefix", dev), _ptr(v_prefix, kv, dt, "v_prefix", dev),
            _ptr(page_meta, (page_meta_size(sh),), torch.uint8, "page_meta", dev),
            _ptr(k_blk, kb, dt, "k_blk", dev), _ptr(v_blk, kb, dt, "v_blk", dev),
            _ptr(o_p, qs, torch.float32, "o_p", dev), _ptr(l_p, rs, torch.float32, "l_p", dev),
            _ptr(out, qs, torch.float32, "out", dev),
            _ptr(out_lse, rs, torch.float32, "out_lse", dev),
            _ptr(active_idx, (sh.num_seqs, sh.n_q_heads, A), torch.int32, "active_idx", dev),
            _ptr(page_idx, (sh.num_seqs, sh.n_q_heads, A, k), torch.int32, "page_idx", dev),
            _ptr(union_count, (sh.num_seqs, sh.n_kv_heads), torch.int32, "union_count", dev)]
    _check(lib().losa_step_noalloc(ctypes.byref(sh), *args, _stream(stream)))


def read_device_status(workspace: torch.Tensor, stream=None) -> int:
    return lib().losa_read_device_status(ctypes.c_void_p(workspace.data_ptr()), _stream(stream))


def noalloc_read_status(stream=None) -> int:
    """Device-side status of the ``losa_step_noalloc`` calls on the current
    device (read and cleared; synchronises the stream)."""
    return lib().losa_noalloc_read_status(_stream(stream))
