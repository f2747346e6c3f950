"""Per-phase timeline of the LoSA step kernel (profiling aid).

Builds (if needed) and loads the tracing copy of the library,
``liblosa_trace.so`` (``build.build(trace=True)``): the same kernels, except
that thread 0 of each CTA stamps ``%globaltimer`` at every phase boundary of
the step.  Runs a few steps of a synthetic workload through the public API
with that library and prints, per phase, the minimum / median / maximum
over the CTAs of the time since the first CTA started (microseconds).

    python -m sparse_long_context_mse_b200.phase_trace [workload ...]

The product library is not touched: this module only imports ``api`` with
its library path pointed at the tracing build, in its own process.
"""
from __future__ import annotations

import ctypes
import statistics
import sys

PHASES = {
    0: "start (after the wait on the previous grid)",
    1: "queries landed",
    2: "locality (per-token MSE) done",
    3: "active set, interval factors, staging done",
    4: "tensor-core A fragments ready",
    5: "metadata stage 0 ready",
    6: "last metadata stage ready",
    7: "last chunk's candidate selection starts",
    8: "candidate lists final (before cluster barrier 1)",
    9: "cluster barrier 1 passed",
    10: "merge done",
    11: "the CTA's page list done (own rows' pages, or its union slots)",
    12: "page gather issued",
    13: "suffix attention done",
    14: "first gathered pages landed",
    15: "page attention done",
    16: "partials final (own rows merged, or cluster barrier 2 passed)",
    17: "outputs written (before the last cluster barrier)",
    18: "end",
    19: "(warp 0, last chunk) survivors of its two rows found",
    20: "(warp 0, last chunk) survivors rescored exactly",
}
for _t in range(8):
    PHASES[24 + _t] = f"stage {_t} ready (thread 0)"
    PHASES[32 + _t] = f"stage {_t} refill issued"
    PHASES[40 + _t] = f"stage {_t} released by warp 4"
K_PHASES, K_CTAS = 48, 512


def _lib():
    from sparse_long_context_mse_b200 import api, build
    api.LIB_PATH = build.build(trace=True)
    L = api.lib()
    L.losa_phase_read.argtypes = [ctypes.c_void_p, ctypes.c_int]
    L.losa_phase_read.restype = ctypes.c_int
    L.losa_phase_clear.argtypes = []
    L.losa_phase_clear.restype = ctypes.c_int
    return api, L


def trace(name: str, reps: int = 3, n_layers: int = 2):
    """Per-phase (min, median, max) microseconds of ``reps`` steps of the
    workload ``name`` (the last rep's table is returned, all are printed)."""
    import torch
    from sparse_long_context_mse_b200 import synth
    api, L = _lib()
    cfg = synth.workload(name)
    dev = torch.device("cuda", 0)
    sh = api.shape_of(cfg, scale=float(1.0 / cfg.head_dim ** 0.5))
    T = cfg.steps
    ws_dense = api.alloc_workspace(sh, api.LOSA_WS_DENSE, dev)
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, dev)
    layers = []
    for li in range(n_layers):
        pre = synth.gen_prefix(cfg, li, device=dev)
        q = synth.gen_queries(cfg, li, steps=T, device=dev, hot_u=pre["hot_u"])["q"]
        kv = [synth.gen_block_kv(cfg, li, t, device=dev) for t in range(T)]
        meta = api.alloc_page_meta(sh, dev)
        api.build_page_meta(sh, pre["k_prefix"], meta)
        rows = (sh.num_seqs, sh.n_q_heads, sh.block_size)
        o_p = torch.empty(*rows, sh.head_dim, device=dev)
        l_p = torch.empty(*rows, device=dev)
        out, lse = torch.empty_like(o_p), torch.empty_like(l_p)
        api.dense_prefix(sh, q[0], pre["k_prefix"], pre["v_prefix"], kv[0][0], kv[0][1], o_p, l_p,
                         out, lse, ws_dense)
        layers.append((pre, q, kv, meta, o_p, l_p, out, lse))

    def step(i):
        pre, q, kv, meta, o_p, l_p, out, lse = layers[i % n_layers]
        t = 1 + i % (T - 1)
        api.step(sh, q[t], q[t - 1], pre["k_prefix"], pre["v_prefix"], meta, kv[t][0], kv[t][1],
                 o_p, l_p, out, lse, ws)

    for i in range(6):  # warm-up
        step(i)
    torch.cuda.synchronize()
    table = None
    for rep in range(reps):
        assert L.losa_phase_clear() == 0
        torch.cuda.synchronize()
        step(rep)
        torch.cuda.synchronize()
        buf = (ctypes.c_ulonglong * (K_CTAS * K_PHASES))()
        assert L.losa_phase_read(ctypes.addressof(buf), K_CTAS * K_PHASES) == 0
        ctas = [[buf[c * K_PHASES + i] for i in range(K_PHASES)] for c in range(K_CTAS)]
        ctas = [r for r in ctas if r[0]]
        t0 = min(r[0] for r in ctas)
        table = {}
        print(f"{name}: step {rep}, {len(ctas)} CTAs (us since the first CTA's start)")
        for i, label in PHASES.items():
            v = [(r[i] - t0) / 1e3 for r in ctas if r[i]]
            if v:
                table[i] = (min(v), statistics.median(v), max(v))
                print(f"  {i:2d} {label:52s} min {min(v):7.2f}  med {statistics.median(v):7.2f}"
                      f"  max {max(v):7.2f}")
    assert api.read_device_status(ws) == 0
    return table


if __name__ == "__main__":
    from sparse_long_context_mse_b200 import synth
    for n in sys.argv[1:] or [synth.GQA64K]:
        trace(n)
