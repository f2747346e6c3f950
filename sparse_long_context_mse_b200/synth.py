"""Seeded synthetic workloads for LoSA per-denoising-step attention.

This module only draws random tensors.  It holds none of the method's
arithmetic (no locality score, no bound, no attention), so both the CUDA path
and the CPU oracle can consume the very same tensors.

Workloads follow the settings the LoSA pages evaluate ("64K context, block
size 16", budgets 128/256, block sizes 16 and 32; LoSA paper, experiments
section) and the locality observation (a few tokens change a lot between
consecutive denoising steps, most barely move; paper, "locality of
representation changes").  The generative recipe, per sequence:

* prefix keys/values and block keys/values ~ N(0, 1);
* a unit "hot" direction u_g per KV head; ``n_hot`` prefix positions drawn
  without replacement get ``k += 4 u_g`` (these are the pages a query that
  leans on u_g should find);
* Q_1 ~ N(0, 1) + 0.5 u_g for every query head of group g;
* Q_t = Q_{t-1} + sigma_stable * N(0, 1) for stable tokens and
  + sigma_active * N(0, 1) for ``n_active`` tokens per query head, drawn
  without replacement and re-drawn every step (the planted active set);
* everything is drawn in fp32, then rounded to the storage dtype (bf16
  round-to-nearest-even); the rounded values are the ground truth.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class LosaConfig:
    name: str
    num_seqs: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    prefix_len: int
    page_size: int
    block_size: int
    n_active: int
    token_budget: int
    dtype: str
    n_hot: int
    sigma_stable: float
    sigma_active: float
    seed: int
    steps: int = 2          # denoising steps generated (Q_1 .. Q_T)
    layers: int = 1
    # per-layer overrides (full-depth stack): list of (n_active, sigma_stable)
    layer_profile: Optional[tuple] = None

    # ---- derived sizes -------------------------------------------------
    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    @property
    def n_pages(self) -> int:
        return (self.prefix_len + self.page_size - 1) // self.page_size

    @property
    def pages_per_row(self) -> int:
        return min(self.token_budget // self.page_size, self.n_pages)

    def for_layer(self, layer: int) -> "LosaConfig":
        """Config seen by one layer of a full-depth stack."""
        if self.layer_profile is None:
            return self
        a, sig = self.layer_profile[layer]
        return dataclasses.replace(self, n_active=a, sigma_stable=sig, layer_profile=None)

    def with_(self, **kw) -> "LosaConfig":
        return dataclasses.replace(self, **kw)

    @property
    def torch_dtype(self):
        return torch.float32 if self.dtype == F32 else torch.bfloat16


def _outer_inner_profile(n_layers=36, outer=4, a_outer=2, s_outer=0.005, a_mid=6, s_mid=0.02):
    prof = []
    for l in range(n_layers):
        if l < outer or l >= n_layers - outer:
            prof.append((a_outer, s_outer))
        else:
            prof.append((a_mid, s_mid))
    return tuple(prof)


#: Workload names: a tiny fp32 single head; one 8B-class GQA layer (32 query,
#: 8 KV heads) at 16K; the same layer at the 64K / B=16 point the pages time;
#: 8 independent 32K sequences with B=32; a 36-layer stack at 128K.
TINY = "tiny_f32_L2048"
GQA16K = "gqa32x8_L16384_B16"
GQA64K = "gqa32x8_L65536_B16"
BATCH8 = "batch8_gqa32x8_L32768_B32"
STACK36 = "stack36_gqa32x8_L131072_B16"

WORKLOADS = {c.name: c for c in (
    LosaConfig(TINY, 1, 1, 1, 128, 2048, 16, 16, 4, 128, F32,
               n_hot=32, sigma_stable=0.01, sigma_active=1.0, seed=0),
    LosaConfig(GQA16K, 1, 32, 8, 128, 16384, 16, 16, 4, 256, BF16,
               n_hot=64, sigma_stable=0.01, sigma_active=1.0, seed=1),
    LosaConfig(GQA64K, 1, 32, 8, 128, 65536, 16, 16, 4, 128, BF16,
               n_hot=64, sigma_stable=0.01, sigma_active=1.0, seed=2, steps=8),
    LosaConfig(BATCH8, 8, 32, 8, 128, 32768, 16, 32, 8, 256, BF16,
               n_hot=327, sigma_stable=0.02, sigma_active=1.0, seed=300),
    LosaConfig(STACK36, 1, 32, 8, 128, 131072, 16, 16, 6, 256, BF16,
               n_hot=64, sigma_stable=0.02, sigma_active=1.0, seed=400, steps=8,
               layers=36, layer_profile=_outer_inner_profile()),
)}


def workload(name: str) -> LosaConfig:
    return WORKLOADS[name]


# ---------------------------------------------------------------------------
# seeding
# ---------------------------------------------------------------------------
_KIND_PREFIX, _KIND_QUERY, _KIND_BLOCK = 1, 2, 3


def seq_seed(cfg: LosaConfig, layer: int, s: int) -> int:
    """Per-sequence seed: 300+s for the batched workload, 400+layer for the
    stack, otherwise the config seed (plus 1000 per extra layer copy)."""
    if cfg.name.startswith("batch8"):
        return cfg.seed + s + 1000 * layer
    if cfg.layer_profile is not None or cfg.name.startswith("stack36"):
        return cfg.seed + layer + 1000 * s
    return cfg.seed + 1000 * layer + 7919 * s


def _gen(seed: int, kind: int, step: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + kind * 10_007 + step) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _randn(shape, g, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _hot_dirs_and_pos(cfg: LosaConfig, seed: int, device):
    g = _gen(seed, _KIND_PREFIX, 0, device)
    u = _randn((cfg.n_kv_heads, cfg.head_dim), g, device)
    u = u / u.norm(dim=-1, keepdim=True)
    n_hot = min(cfg.n_hot, cfg.prefix_len)
    pos = torch.stack([
        torch.randperm(cfg.prefix_len, generator=g, device=device)[:n_hot]
        for _ in range(cfg.n_kv_heads)
    ])
    return u, pos


def gen_prefix(cfg: LosaConfig, layer: int = 0, device="cpu"):
    """Prefix K/V ``[S][Hkv][L][d]`` in the storage dtype, plus the hot
    directions ``u [S][Hkv][d]`` (fp32) and hot positions ``[S][Hkv][n_hot]``."""
    ks, vs, us, ps = [], [], [], []
    for s in range(cfg.num_seqs):
        seed = seq_seed(cfg, layer, s)
        u, pos = _hot_dirs_and_pos(cfg, seed, device)
        g = _gen(seed, _KIND_PREFIX, 1, device)
        k = _randn((cfg.n_kv_heads, cfg.prefix_len, cfg.head_dim), g, device)
        v = _randn((cfg.n_kv_heads, cfg.prefix_len, cfg.head_dim), g, device)
        for h in range(cfg.n_kv_heads):
            k[h, pos[h]] += 4.0 * u[h]
        ks.append(k.to(cfg.torch_dtype))
        vs.append(v.to(cfg.torch_dtype))
        us.append(u)
        ps.append(pos)
    return {"k_prefix": torch.stack(ks).contiguous(), "v_prefix": torch.stack(vs).contiguous(),
            "hot_u": torch.stack(us), "hot_pos": torch.stack(ps)}


def gen_block_kv(cfg: LosaConfig, layer: int = 0, step: int = 0, device="cpu"):
    """Block keys/values ``[S][Hkv][B][d]``.  A diffusion LM recomputes them
    every denoising step, so each step draws a fresh pair."""
    ks, vs = [], []
    for s in range(cfg.num_seqs):
        g = _gen(seq_seed(cfg, layer, s), _KIND_BLOCK, step, device)
        ks.append(_randn((cfg.n_kv_heads, cfg.block_size, cfg.head_dim), g, device))
        vs.append(_randn((cfg.n_kv_heads, cfg.block_size, cfg.head_dim), g, device))
    return (torch.stack(ks).to(cfg.torch_dtype).contiguous(),
            torch.stack(vs).to(cfg.torch_dtype).contiguous())


def gen_queries(cfg: LosaConfig, layer: int = 0, steps: Optional[int] = None, device="cpu",
                hot_u: Optional[torch.Tensor] = None):
    """Queries for ``steps`` consecutive denoising steps.

    Returns ``{"q": [Q_1, ..., Q_T]`` (each ``[S][Hq][B][d]`` in the storage
    dtype) and ``"planted": [P_2, ..., P_T]`` (bool ``[S][Hq][B]``: tokens
    given the large drift between step t-1 and t)}.
    """
    steps = cfg.steps if steps is None else steps
    G = cfg.group
    per_seq_q: List[List[torch.Tensor]] = []
    per_seq_planted: List[List[torch.Tensor]] = []
    for s in range(cfg.num_seqs):
        seed = seq_seed(cfg, layer, s)
        if hot_u is None:
            u, _ = _hot_dirs_and_pos(cfg, seed, device)
        else:
            u = hot_u[s].to(device)
        g = _gen(seed, _KIND_QUERY, 0, device)
        q = _randn((cfg.n_q_heads, cfg.block_size, cfg.head_dim), g, device)
        q = q + 0.5 * u.repeat_interleave(G, dim=0)[:, None, :]
        qs = [q.clone()]
        planted = []
        for t in range(1, steps):
            g = _gen(seed, _KIND_QUERY, t, device)
            drift = _randn((cfg.n_q_heads, cfg.block_size, cfg.head_dim), g, device)
            act = torch.zeros((cfg.n_q_heads, cfg.block_size), dtype=torch.bool, device=device)
            for h in range(cfg.n_q_heads):
                idx = torch.randperm(cfg.block_size, generator=g, device=device)[:cfg.n_active]
                act[h, idx] = True
            sig = torch.where(act, torch.tensor(cfg.sigma_active, device=device),
                              torch.tensor(cfg.sigma_stable, device=device))
            q = q + sig[..., None] * drift
            qs.append(q.clone())
            planted.append(act)
        per_seq_q.append(qs)
        per_seq_planted.append(planted)
    q_out = [torch.stack([per_seq_q[s][t] for s in range(cfg.num_seqs)]).to(cfg.torch_dtype).contiguous()
             for t in range(steps)]
    p_out = [torch.stack([per_seq_planted[s][t] for s in range(cfg.num_seqs)])
             for t in range(steps - 1)]
    return {"q": q_out, "planted": p_out}

