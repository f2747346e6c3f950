"""Exact ties on the GPU: integer-valued queries, keys and values (small
integers, exact in bf16 and in every fp32 product and partial sum), so that
many tokens share one locality score and many pages share one bound.  The
selection rule breaks each tie to the lower token / page index (LoSA paper,
methodology: locality pruning and QUEST page selection); the CUDA path must
take exactly the oracle's active sets, page lists and union sizes, with no
tolerance at all."""
import zlib

import numpy as np
import pytest
import torch

import oracle
from losa_testutil import (DEV, Case, check_meta, check_step_full, gpu_dense, gpu_meta,
                           gpu_step, oshape, scale_of)
from sparse_long_context_mse_b200 import api

pytestmark = pytest.mark.gpu

SHAPES = {
    # name: (S, Hq, Hkv, L, B, A, budget)
    "ragged": (3, 6, 2, 1000, 5, 2, 48),
    "gqa32x8": (1, 32, 8, 4096, 16, 4, 128),
    "B32_G4": (2, 8, 2, 2500, 32, 8, 256),
}


def integer_case(S, Hq, Hkv, L, B, A, budget, seed, kmag=4):
    g = torch.Generator().manual_seed(seed)
    d = 128
    ri = lambda lo, hi, *s: torch.randint(lo, hi + 1, s, generator=g).float()
    qp = ri(-4, 4, S, Hq, B, d)
    # each token changes by +-1 on 0, 1 or 2 channels: its mse is 0, 1/128 or
    # 2/128, so most of a head's tokens tie with others at the |A|-th place
    qc = qp.clone()
    nchg = torch.randint(0, 3, (S, Hq, B), generator=g)
    for s in range(S):
        for h in range(Hq):
            for t in range(B):
                ch = torch.randperm(d, generator=g)[: int(nchg[s, h, t])]
                qc[s, h, t, ch] += torch.where(torch.rand(len(ch), generator=g) < 0.5, -1.0, 1.0)
    c = Case.__new__(Case)
    c.cfg = None
    c.layer = 0
    c.sh = api.make_shape(S, Hq, Hkv, d, L, 16, B, A, budget, "bf16", scale=scale_of(d))
    # keys with a small range: most pages' per-channel min and max coincide,
    # so most pages share one bound
    c.K = ri(-kmag, kmag, S, Hkv, L, d).to(torch.bfloat16).to(DEV)
    c.V = ri(-4, 4, S, Hkv, L, d).to(torch.bfloat16).to(DEV)
    c.q = [qp.to(torch.bfloat16).to(DEV), qc.to(torch.bfloat16).to(DEV)]
    c.kb = [ri(-4, 4, S, Hkv, B, d).to(torch.bfloat16).to(DEV) for _ in range(2)]
    c.vb = [ri(-4, 4, S, Hkv, B, d).to(torch.bfloat16).to(DEV) for _ in range(2)]
    c.planted = None
    c._host = {}
    return c


@pytest.mark.parametrize("kmag", [1, 4])
@pytest.mark.parametrize("name", sorted(SHAPES))
def test_integer_ties_are_exact(name, kmag):
    S, Hq, Hkv, L, B, A, budget = SHAPES[name]
    c = integer_case(S, Hq, Hkv, L, B, A, budget, seed=zlib.crc32(name.encode()) % 1000 + kmag,
                     kmag=kmag)
    sh = c.sh
    meta = gpu_meta(sh, c.K)
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    # the step is checked on its own: the oracle starts from the GPU's cache
    # (the cold-start pass rounds its weights to bf16, which with values of
    # magnitude 4 alone moves outputs by up to ~4 * 2^-9)
    cache_o = {"o_p": oracle.f32(cache_g["o_p"]), "l_p": oracle.f32(cache_g["l_p"])}
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1], cache_g["o_p"],
                   cache_g["l_p"])
    # the ties are really there (else this test would prove nothing)
    r = oracle.step(oshape(sh), c.q[1], c.q[0], c.host("K"), c.host("V"), kmin, kmax, c.kb[1],
                    c.vb[1], cache_o["o_p"], cache_o["l_p"], want_bound=True)
    mse = r["mse"]
    tied_heads = sum(1 for s in range(S) for h in range(Hq)
                     if np.sort(mse[s, h])[::-1][A - 1] == np.sort(mse[s, h])[::-1][A])
    k = sh.pages_per_row
    tied_rows = sum(1 for s in range(S) for h in range(Hq) for a in range(A)
                    if np.sort(r["bound"][s, h, a])[::-1][k - 1] == np.sort(r["bound"][s, h, a])[::-1][k])
    assert tied_heads > 0 and tied_rows > 0, (tied_heads, tied_rows)
    check_step_full(c, 1, res, cache_o, kmin, kmax, tag=f"ties/{name}/{kmag}")
    assert api.read_device_status(res["ws"]) == api.LOSA_OK
