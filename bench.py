#!/usr/bin/env python
"""Benchmark of LoSA per-denoising-step attention on B200.

Workload: one 8B-class GQA attention layer (32 query / 8 KV heads, head_dim
128, bf16) at a 65536-token prefix, block 16, |A| = 4 per head, budget 128
tokens (8 pages of 16), i.e. the "64K context, block size 16" point the LoSA
pages time.  A step is one LoSA denoising step of one layer: locality score
and active set, bound scoring and page selection, union gather, suffix,
merge, cache write-back.

The timed loop replays a CUDA graph of consecutive steps over ``--layers``
distinct layer copies (prefix K/V, page metadata, cache, queries), so the
bytes touched between two visits of a layer exceed the 126 MB L2: every step
reads its metadata and pages from HBM.

One JSON line on stdout (rank 0).  ``--impl reference`` times the CPU oracle
instead (bounded sample, host cores).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LoSA attention steps/s and achieved HBM GB/s (frac of peak) at 64K ctx, B=16"
UNIT = "steps/s"
WORKLOAD = "gqa32x8_L65536_B16"  # the 64K-context, B=16 layer


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=8000)
    ap.add_argument("--warmup", type=int, default=160)
    ap.add_argument("--impl", choices=["losa", "reference"], default="losa")
    ap.add_argument("--layers", type=int, default=16, help="distinct layer copies rotated")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the block / dense / e2e / oracle side measurements")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing (independent replicas: no collective in the data path)
# ---------------------------------------------------------------------------
def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    """The largest value of x over the ranks (every rank takes part)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, steps_per_rank, ms_max):
    """Whole-job steps/s: each of `world` replicas ran `steps_per_rank` steps,
    and the job took as long as its slowest rank."""
    return world * steps_per_rank / (ms_max / 1e3)


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, the source nvidia-smi reads)
# ---------------------------------------------------------------------------
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
            0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
            0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, cuda_index, period_s=0.005):
        self.samples, self.reasons, self.max_mhz = [], 0, None
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            idx = torch.cuda._get_nvml_device_index(cuda_index)
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 -- no NVML: report without clocks
            self.err = repr(e)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        reasons = [n for b, n in _REASONS.items() if self.reasons & b and b != 0x1]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# peaks, roofline bytes
# ---------------------------------------------------------------------------
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the sources the two step kernels are compiled from (their launch code and
# shared headers included)
STEP_SOURCES = ("step_fused.cu", "step.cu", "losa_common.cuh", "ptx.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "sparse_long_context_mse_b200", "csrc")
    for path in [os.path.join(csrc, n) for n in STEP_SOURCES] + [
            os.path.join(ROOT, "include", "losa.h")]:
        with open(path, "rb") as f:
            h.update(os.path.basename(path).encode() + f.read())
    return h.hexdigest()[:16]


def committed_traffic():
    """DRAM bytes per step from the committed ncu summary, if it was taken on
    the current kernel sources."""
    p = os.path.join(ROOT, "profiles", "traffic_losa_step_64k.json")
    try:
        with open(p) as f:
            j = json.load(f)
        if j.get("kernel_source_hash") == kernel_source_hash():
            return float(j["dram_bytes_per_step"])
    except (OSError, ValueError, KeyError):
        pass
    return None


def step_bytes(sh, union_counts, esz):
    """Algorithmic bytes of one LoSA step: metadata scan + union K/V pages +
    Q_cur/Q_prev + cached o_p/L_p read + active-row write-back."""
    S, Hq, Hkv, d, B, A = (sh.num_seqs, sh.n_q_heads, sh.n_kv_heads, sh.head_dim,
                           sh.block_size, sh.n_active)
    P, ps = sh.n_pages, sh.page_size
    meta = S * Hkv * P * 2 * d * esz
    union = int(sum(union_counts)) * ps * d * 2 * esz
    q = 2 * S * Hq * B * d * esz
    cache_r = S * Hq * B * (d + 1) * 4
    cache_w = S * Hq * A * (d + 1) * 4
    return meta + union + q + cache_r + cache_w


def launches_per_step(sh):
    """Kernels one losa_step launches: the scan and gather kernels always, the
    combine kernel whenever some query row is active."""
    return 3 if sh.n_active > 0 else 2


# ---------------------------------------------------------------------------
# the CUDA path
# ---------------------------------------------------------------------------
class Layer:
    pass


def build_layers(cfg, n_layers, dev):
    import torch
    from sparse_long_context_mse_b200 import api, synth
    sh = api.shape_of(cfg, scale=float(1.0 / cfg.head_dim ** 0.5))
    T = cfg.steps
    layers = []
    ws_dense = api.alloc_workspace(sh, api.LOSA_WS_DENSE, dev)
    for li in range(n_layers):
        L = Layer()
        pre = synth.gen_prefix(cfg, li, device=dev)
        L.K, L.V = pre["k_prefix"], pre["v_prefix"]
        L.q = synth.gen_queries(cfg, li, steps=T, device=dev, hot_u=pre["hot_u"])["q"]
        L.kb, L.vb = zip(*[synth.gen_block_kv(cfg, li, t, device=dev) for t in range(T)])
        L.meta = api.alloc_page_meta(sh, dev)
        api.build_page_meta(sh, L.K, L.meta)
        rows = (sh.num_seqs, sh.n_q_heads, sh.block_size)
        L.o_p = torch.empty(*rows, sh.head_dim, device=dev)
        L.l_p = torch.empty(*rows, device=dev)
        L.out = torch.empty_like(L.o_p)
        L.lse = torch.empty_like(L.l_p)
        api.dense_prefix(sh, L.q[0], L.K, L.V, L.kb[0], L.vb[0], L.o_p, L.l_p, L.out, L.lse,
                         ws_dense)
        L.ucount = torch.zeros(sh.num_seqs, sh.n_kv_heads, dtype=torch.int32, device=dev)
        layers.append(L)
    torch.cuda.synchronize()
    return sh, layers, ws_dense


def run_losa(args):
    import torch
    from sparse_long_context_mse_b200 import api, synth
    rank, world, local = dist_setup(args)
    dev = torch.device("cuda", local)
    cfg = synth.workload(WORKLOAD)
    T = cfg.steps
    sh, layers, ws_dense = build_layers(cfg, args.layers, dev)
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, dev)
    nL = len(layers)
    # schedule: step j of a graph replay runs layer j % nL with query pair
    # (t, t-1), t cycling through the block's LoSA steps 1..T-1
    sched = [(j % nL, 1 + (j // nL) % (T - 1)) for j in range(nL * (T - 1))]
    stream = torch.cuda.Stream(device=dev)

    def one_step(li, t, want_union=False):
        L = layers[li]
        api.step(sh, L.q[t], L.q[t - 1], L.K, L.V, L.meta, L.kb[t], L.vb[t], L.o_p, L.l_p,
                 L.out, L.lse, ws, union_count=L.ucount if want_union else None, stream=stream)

    # union counts of every scheduled step (untimed): the measured U of the roofline
    ubytes = []
    with torch.cuda.stream(stream):
        for li, t in sched:
            one_step(li, t, want_union=True)
            ubytes.append(layers[li].ucount.sum().item())
    torch.cuda.synchronize()
    esz = 2
    bytes_sched = [step_bytes(sh, [u], esz) for u in ubytes]
    union_per_kv = [u / (sh.num_seqs * sh.n_kv_heads) for u in ubytes]

    # capture one pass over the schedule
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        for li, t in sched[:4]:
            one_step(li, t)
    stream.synchronize()
    with torch.cuda.graph(graph, stream=stream):
        for li, t in sched:
            one_step(li, t)
    per_replay = len(sched)
    warm_replays = max(3, -(-args.warmup // per_replay))
    replays = max(1, -(-args.steps // per_replay))
    steps_timed = replays * per_replay
    # graph.replay() launches on the current stream: keep it `stream`, the
    # stream the events are recorded on
    with torch.cuda.stream(stream):
        for _ in range(warm_replays):
            graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk, torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(replays):
            graph.replay()
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms = ev0.elapsed_time(ev1)
    ms_max = max_over_ranks(ms, world)
    ms_per_step = ms_max / steps_timed
    value = job_throughput(world, steps_timed, ms_max)
    bytes_per_step = sum(bytes_sched) / len(bytes_sched)
    achieved = bytes_per_step / (ms_per_step / 1e3) / 1e9
    peak, peak_kind = measured_peaks()

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": steps_timed, "warmup": warm_replays * per_replay,
        "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator: N(0,1) K/V with hot pages, planted active tokens)",
        "config": {"workload": cfg.name, "num_seqs": sh.num_seqs, "n_q_heads": sh.n_q_heads,
                   "n_kv_heads": sh.n_kv_heads, "head_dim": sh.head_dim,
                   "prefix_len": sh.prefix_len, "page_size": sh.page_size,
                   "block_size": sh.block_size, "n_active": sh.n_active,
                   "token_budget": sh.token_budget, "layers_rotated": nL,
                   "l2": f"inputs larger than L2: {nL} layer copies rotated "
                         f"(~{bytes_per_step * nL / 1e6:.0f} MB touched per rotation)",
                   "timing": "CUDA graph of consecutive steps, CUDA events on the launch stream"},
        "us_per_layer_step": ms_per_step * 1e3,
        "union_pages_per_kv_head": {"mean": statistics.mean(union_per_kv),
                                    "min": min(union_per_kv), "max": max(union_per_kv),
                                    "density": statistics.mean(union_per_kv) / sh.n_pages},
        "roofline": {"bound": "hbm", "kernel": "losa_step (all launches of one step)",
                     "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                     "algorithmic_bytes_per_step": round(bytes_per_step),
                     "traffic": committed_traffic()},
        "gpu_launches": steps_timed * launches_per_step(sh),
        "clocks": clk.summary(),
    }
    if not args.no_extras:
        res.update(extras(args, sh, layers, ws, ws_dense, stream, dev, world, sched))
        res["naive_quest_all_B"] = naive_quest(stream, dev, world,
                                               statistics.mean(union_per_kv), ms_per_step)
        res["block"]["losa_vs_dense_step_speedup"] = round(
            res["dense_step_us"] / res["us_per_layer_step"], 3)
    if rank == 0:
        print(json.dumps(res), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def naive_quest(stream, dev, world, losa_union, losa_ms):
    """The same kernels with every block token active (|A| = B): QUEST page
    selection for all B queries, the baseline LoSA's locality pruning is
    measured against.  Reports the union (KV pages loaded per KV head), its
    inflation over LoSA's, and the step time."""
    import dataclasses
    import torch
    from sparse_long_context_mse_b200 import api, synth
    cfg = synth.workload(WORKLOAD)
    cfg = dataclasses.replace(cfg, n_active=cfg.block_size)
    n_layers = 2  # 2 x ~280 MB of prefix K/V + metadata: larger than L2
    sh, layers, _ = build_layers(cfg, n_layers, dev)
    ws = api.alloc_workspace(sh, api.LOSA_WS_STEP, dev)
    T = cfg.steps
    sched = [(li, t) for t in range(1, T) for li in range(n_layers)]
    unions = []
    with torch.cuda.stream(stream):
        for li, t in sched:
            L = layers[li]
            api.step(sh, L.q[t], L.q[t - 1], L.K, L.V, L.meta, L.kb[t], L.vb[t], L.o_p, L.l_p,
                     L.out, L.lse, ws, union_count=L.ucount, stream=stream)
            unions.append(L.ucount.sum().item() / (sh.num_seqs * sh.n_kv_heads))
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for li, t in sched:
            L = layers[li]
            api.step(sh, L.q[t], L.q[t - 1], L.K, L.V, L.meta, L.kb[t], L.vb[t], L.o_p, L.l_p,
                     L.out, L.lse, ws, stream=stream)
    reps = 20
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world) / (reps * len(sched))
    del g
    u = statistics.mean(unions)
    return {"n_active": cfg.n_active, "union_pages_per_kv_head": round(u, 2),
            "density": round(u / sh.n_pages, 5), "us_per_step": round(ms * 1e3, 3),
            "union_vs_losa": round(u / losa_union, 3), "step_time_vs_losa": round(ms / losa_ms, 3)}


def extras(args, sh, layers, ws, ws_dense, stream, dev, world, sched):
    """Side measurements: cold-start dense step, T=8 block, end-to-end with
    host buffers, oracle CPU baseline."""
    import torch
    from sparse_long_context_mse_b200 import api
    out = {}
    T = len(layers[0].q)
    nL = len(layers)

    def time_graph(fn, reps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.stream(stream):
            fn()
        stream.synchronize()
        with torch.cuda.graph(g, stream=stream):
            fn()
        with torch.cuda.stream(stream):
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
        torch.cuda.synchronize()
        ms = max_over_ranks(e0.elapsed_time(e1), world) / reps
        del g
        return ms

    def dense_all():
        for L in layers:
            api.dense_prefix(sh, L.q[0], L.K, L.V, L.kb[0], L.vb[0], L.o_p, L.l_p, L.out, L.lse,
                             ws_dense, stream=stream)

    def block_all():
        for L in layers:
            api.dense_prefix(sh, L.q[0], L.K, L.V, L.kb[0], L.vb[0], L.o_p, L.l_p, L.out, L.lse,
                             ws_dense, stream=stream)
            for t in range(1, T):
                api.step(sh, L.q[t], L.q[t - 1], L.K, L.V, L.meta, L.kb[t], L.vb[t], L.o_p,
                         L.l_p, L.out, L.lse, ws, stream=stream)

    # the two step variants on the same schedule: every active row over its
    # group's whole union; drift-safe locality against per-row references
    import copy
    sh_u = copy.copy(sh)
    sh_u.flags = api.LOSA_STEP_ATTEND_UNION
    q_ref = [L.q[0].clone() for L in layers]

    def union_all():
        for li, t in sched:
            L = layers[li]
            api.step(sh_u, L.q[t], L.q[t - 1], L.K, L.V, L.meta, L.kb[t], L.vb[t], L.o_p, L.l_p,
                     L.out, L.lse, ws, stream=stream)

    def ref_all():
        for li, t in sched:
            L = layers[li]
            api.step_ref(sh, L.q[t], q_ref[li], L.K, L.V, L.meta, L.kb[t], L.vb[t], L.o_p,
                         L.l_p, L.out, L.lse, ws, stream=stream)

    out["variants"] = {
        "attend_union_us_per_step": round(time_graph(union_all, 10) / len(sched) * 1e3, 3),
        "drift_safe_us_per_step": round(time_graph(ref_all, 10) / len(sched) * 1e3, 3)}

    # prefix growth: a committed block appended inside the buffers' capacity
    # (one layer copy with room for one more block; the same append repeated)
    import copy as _copy
    L0 = layers[0]
    sh_a = _copy.copy(sh)
    sh_a.prefix_capacity = sh.prefix_len + sh.block_size
    Kc = torch.empty(sh.num_seqs, sh.n_kv_heads, sh_a.prefix_capacity, sh.head_dim,
                     dtype=L0.K.dtype, device=dev)
    Vc = torch.empty_like(Kc)
    Kc[:, :, :sh.prefix_len] = L0.K
    Vc[:, :, :sh.prefix_len] = L0.V
    meta_c = api.alloc_page_meta(sh_a, dev)
    api.build_page_meta(sh_a, Kc, meta_c, stream=stream)

    def append_one():
        api.append_block(sh_a, L0.kb[0], L0.vb[0], Kc, Vc, meta_c, stream=stream)

    out["append_block_us"] = round(time_graph(append_one, 50) * 1e3, 3)
    del Kc, Vc, meta_c

    # a variable-length batch: four sequences of 1, 1/2, 1/4 and 1/8 (+5
    # tokens) of the prefix length in one call, against the same batch with
    # every sequence at the longest length; NC copies rotated so that the
    # bytes of a rotation exceed L2
    lens = [sh.prefix_len, sh.prefix_len // 2, sh.prefix_len // 4, sh.prefix_len // 8 + 5]
    S4, NC = len(lens), 4
    lens_t = torch.tensor(lens, dtype=torch.int32, device=dev)
    geo = (S4, sh.n_q_heads, sh.n_kv_heads, sh.head_dim, sh.prefix_len, sh.page_size,
           sh.block_size, sh.n_active, sh.token_budget, sh.dtype)
    sh_v = api.make_shape(*geo, scale=sh.scale, prefix_lens=lens_t)
    sh_f = api.make_shape(*geo, scale=sh.scale)

    def rep(t):
        return t.repeat(S4, *([1] * (t.dim() - 1)))

    copies = []
    for _ in range(NC):
        K4, V4 = rep(L0.K), rep(L0.V)
        mv, mf = api.alloc_page_meta(sh_v, dev), api.alloc_page_meta(sh_f, dev)
        api.build_page_meta(sh_v, K4, mv, stream=stream)
        api.build_page_meta(sh_f, K4, mf, stream=stream)
        copies.append((K4, V4, mv, mf))
    q1, q0, kb4, vb4 = rep(L0.q[1]), rep(L0.q[0]), rep(L0.kb[1]), rep(L0.vb[1])
    o_p4 = torch.zeros(S4, sh.n_q_heads, sh.block_size, sh.head_dim, device=dev)
    l_p4 = torch.zeros(S4, sh.n_q_heads, sh.block_size, device=dev)
    out4, lse4 = torch.empty_like(o_p4), torch.empty_like(l_p4)
    ws_v = api.alloc_workspace(sh_v, api.LOSA_WS_STEP, dev)
    ws_f = api.alloc_workspace(sh_f, api.LOSA_WS_STEP, dev)

    def batch_steps(shx, wsx, varlen):
        def run():
            for K4, V4, mv, mf in copies:
                api.step(shx, q1, q0, K4, V4, mv if varlen else mf, kb4, vb4, o_p4, l_p4, out4,
                         lse4, wsx, stream=stream)
        return run

    us_v = time_graph(batch_steps(sh_v, ws_v, True), 10) / NC * 1e3
    us_f = time_graph(batch_steps(sh_f, ws_f, False), 10) / NC * 1e3
    out["varlen_batch"] = {"prefix_lens": lens, "us_per_step": round(us_v, 3),
                           "all_at_longest_us_per_step": round(us_f, 3),
                           "device_status": api.read_device_status(ws_v)}
    del copies

    dense_ms = time_graph(dense_all, 3) / nL
    block_ms = time_graph(block_all, 3) / nL
    out["dense_step_us"] = dense_ms * 1e3
    # the cold-start dense pass against the HBM roofline: the whole prefix's
    # K and V once, the block's queries, the cache and output rows written
    esz = 2
    rows = sh.num_seqs * sh.n_q_heads * sh.block_size
    dense_bytes = (2 * sh.num_seqs * sh.n_kv_heads * sh.prefix_len * sh.head_dim * esz
                   + rows * sh.head_dim * esz + 2 * rows * (sh.head_dim + 1) * 4)
    peak, peak_kind = measured_peaks()
    achieved = dense_bytes / (dense_ms / 1e3) / 1e9
    out["dense_roofline"] = {"bound": "hbm", "kernel": "losa_dense_prefix (tcgen05 pass + split combine)",
                             "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                             "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                             "algorithmic_bytes": dense_bytes}
    out["block"] = {"T": T, "block_us": block_ms * 1e3,
                    "steps_per_s_over_block": T / (block_ms / 1e3),
                    "losa_vs_dense_step_speedup": None}

    # end to end through the public API with host buffers: per step, copy the
    # step's inputs (q_cur, k_blk, v_blk) from pinned host memory, run the
    # step, read the output back
    L0 = layers[0]
    hq = [t.cpu().pin_memory() for t in L0.q]
    hk = [t.cpu().pin_memory() for t in L0.kb]
    hv = [t.cpu().pin_memory() for t in L0.vb]
    dq = [torch.empty_like(t) for t in L0.q]
    dk, dv = torch.empty_like(L0.kb[0]), torch.empty_like(L0.vb[0])
    hout = torch.empty(L0.out.shape, dtype=torch.float32).pin_memory()
    for t in range(T):
        dq[t].copy_(L0.q[t])
    n_e2e = 400
    h2d = dq[0].numel() * dq[0].element_size() + 2 * dk.numel() * dk.element_size()
    d2h = hout.numel() * hout.element_size()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        for i in range(n_e2e + 20):
            if i == 20:
                e0.record(stream)
            t = 1 + i % (T - 1)
            dq[t].copy_(hq[t], non_blocking=True)
            dk.copy_(hk[t], non_blocking=True)
            dv.copy_(hv[t], non_blocking=True)
            api.step(sh, dq[t], dq[t - 1], L0.K, L0.V, L0.meta, dk, dv, L0.o_p, L0.l_p, L0.out,
                     L0.lse, ws, stream=stream)
            hout.copy_(L0.out, non_blocking=True)
        e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / n_e2e
    out["e2e"] = {"value": round(world / (e2e_ms / 1e3), 1), "unit": UNIT,
                  "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                  "note": "public API per step: pinned H2D of q_cur/k_blk/v_blk, losa_step, "
                          "D2H of out; no graph"}
    if int(os.environ.get("RANK", "0")) == 0 and world == 1:
        out["cpu_baseline"] = oracle_baseline(sh, L0, budget_s=12.0)
    return out


# ---------------------------------------------------------------------------
# the oracle (CPU baseline / reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_setup(name=WORKLOAD, device="cpu", layer0=None):
    """Host arrays of one layer of the workload, restricted to query head 0
    and its KV head (1/Hq of a step's rows; the step's work is uniform over
    heads).  The incoming cache is zeros: the step's cost does not depend on
    its values."""
    import numpy as np
    import oracle
    from sparse_long_context_mse_b200 import synth
    cfg = synth.workload(name)
    if layer0 is None:
        pre = synth.gen_prefix(cfg, 0, device=device)
        q = synth.gen_queries(cfg, 0, steps=2, device=device, hot_u=pre["hot_u"])["q"]
        kb, vb = synth.gen_block_kv(cfg, 0, 1, device=device)
        K, V = pre["k_prefix"], pre["v_prefix"]
    else:
        K, V, q, kb, vb = layer0.K, layer0.V, layer0.q, layer0.kb[1], layer0.vb[1]
    sub = cfg.with_(n_q_heads=1, n_kv_heads=1)
    osh = oracle.shape_of(sub, scale=float(np.float32(1.0 / np.sqrt(cfg.head_dim))))
    x = {"Qc": oracle.f32(q[1][:, :1]), "Qp": oracle.f32(q[0][:, :1]),
         "K": oracle.f32(K[:, :1]), "V": oracle.f32(V[:, :1]),
         "Kb": oracle.f32(kb[:, :1]), "Vb": oracle.f32(vb[:, :1])}
    x["kmin"], x["kmax"] = oracle.build_meta(osh, x["K"])
    x["o_p"] = np.zeros((sub.num_seqs, 1, sub.block_size, sub.head_dim), np.float32)
    x["l_p"] = np.zeros((sub.num_seqs, 1, sub.block_size), np.float32)
    return cfg, osh, x


def oracle_sample_step(osh, x):
    import oracle
    oracle.step(osh, x["Qc"], x["Qp"], x["K"], x["V"], x["kmin"], x["kmax"], x["Kb"], x["Vb"],
                x["o_p"], x["l_p"])


def oracle_baseline(sh, layer0, budget_s=12.0):
    cfg, osh, x = oracle_sample_setup(layer0=layer0)
    oracle_sample_step(osh, x)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < budget_s:
        oracle_sample_step(osh, x)
        n += 1
    dt = (time.perf_counter() - t0) / n
    full = dt * sh.n_q_heads
    return {"value": round(1.0 / full, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} oracle steps of query head 0 of layer 0 (1/{sh.n_q_heads} of a step's "
                      f"rows, incl. the full metadata scan of its KV head), scaled x"
                      f"{sh.n_q_heads}; single-threaded C"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cfg, osh, x = oracle_sample_setup()
    for _ in range(max(args.warmup, 0)):
        oracle_sample_step(osh, x)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(osh, x)
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    full = dt * cfg.n_q_heads
    value = 1.0 / full
    sample = (f"each step: the oracle's LoSA step on query head 0 of the 64K workload "
              f"(1/{cfg.n_q_heads} of a step's rows), scaled x{cfg.n_q_heads}; "
              f"single-threaded C")
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
           "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
           "ms_per_step": full * 1e3, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f32", "data": "synthetic",
           "config": {"workload": cfg.name, "prefix_len": cfg.prefix_len,
                      "block_size": cfg.block_size, "n_active": cfg.n_active,
                      "token_budget": cfg.token_budget},
           "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                            "sample": sample},
           "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_losa(args)


if __name__ == "__main__":
    main()
