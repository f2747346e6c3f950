"""Prefix growth on the GPU: losa_append_block commits a finished block to
the prefix inside the buffers' capacity and rebuilds the page records it
touches; every kernel then reads the capacity-strided buffers.  Checked
against the oracle's concatenation and its metadata build, and by running the
dense pass and a LoSA step on the grown prefix."""
import numpy as np
import pytest
import torch

import oracle
from losa_testutil import (DEV, TOL, check_meta, check_step_full, gpu_dense, gpu_meta, gpu_step,
                           maxabs, oshape, random_case)
from sparse_long_context_mse_b200 import api

pytestmark = pytest.mark.gpu

FILL = 7.0  # the unused capacity tail: never read, never written


def _grow_case(dtype, L0, appends, seed):
    S, Hq, Hkv, B, A, budget, d = 2, 8, 2, 16, 4, 64, 128
    c = random_case(S, Hq, Hkv, L0, B, A, budget, dtype, seed=seed)
    Lc = L0 + appends * B + 5
    tdt = c.K.dtype
    K = torch.full((S, Hkv, Lc, d), FILL, dtype=tdt, device=DEV)
    V = torch.full((S, Hkv, Lc, d), FILL, dtype=tdt, device=DEV)
    K[:, :, :L0] = c.K
    V[:, :, :L0] = c.V
    sh = api.make_shape(S, Hq, Hkv, d, L0, 16, B, A, budget, dtype, scale=c.sh.scale,
                        prefix_capacity=Lc)
    meta = api.alloc_page_meta(sh, DEV)
    api.build_page_meta(sh, K, meta)
    Kh, Vh = oracle.f32(c.K), oracle.f32(c.V)
    g = torch.Generator(device="cpu").manual_seed(seed + 100)
    for _ in range(appends):
        kb = torch.randn(S, Hkv, B, d, generator=g).to(tdt).to(DEV)
        vb = torch.randn(S, Hkv, B, d, generator=g).to(tdt).to(DEV)
        api.append_block(sh, kb, vb, K, V, meta)
        Kh, Vh = oracle.append_block(Kh, Vh, kb, vb)
        sh.prefix_len += B
        L = sh.prefix_len
        torch.cuda.synchronize()
        assert np.array_equal(oracle.f32(K[:, :, :L]).view(np.uint32), Kh.view(np.uint32))
        assert np.array_equal(oracle.f32(V[:, :, :L]).view(np.uint32), Vh.view(np.uint32))
        assert bool((K[:, :, L:] == FILL).all()) and bool((V[:, :, L:] == FILL).all())
        check_meta(sh, meta, Kh)  # bit-exact against a rebuild over the grown prefix
    c.sh, c.K, c.V = sh, K, V
    c._host = {"K": Kh, "V": Vh}
    return c, meta


@pytest.mark.parametrize("dtype,L0", [("bf16", 1000), ("f32", 992), ("bf16", 8)])
def test_append_block_matches_rebuild(dtype, L0):
    _grow_case(dtype, L0, 3, seed=11)


def test_append_without_room_is_refused():
    sh = api.make_shape(1, 4, 2, 128, 100, 16, 16, 2, 32, "bf16", prefix_capacity=115)
    t = lambda L: torch.zeros(1, 2, L, 128, dtype=torch.bfloat16, device=DEV)
    meta = api.alloc_page_meta(sh, DEV)
    with pytest.raises(api.LosaError):
        api.append_block(sh, t(16), t(16), t(115), t(115), meta)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_dense_and_step_on_grown_prefix(dtype):
    c, meta = _grow_case(dtype, 1000, 2, seed=12)
    sh = c.sh
    kmin, kmax = check_meta(sh, meta, c.host("K"))
    cache_g = gpu_dense(sh, c.q[0], c.K, c.V, c.kb[0], c.vb[0])
    cache_o = oracle.dense_prefix(oshape(sh), c.q[0], c.host("K"), c.host("V"), c.kb[0], c.vb[0])
    for k in ("o_p", "l_p", "out", "lse"):
        assert maxabs(cache_g[k].cpu().numpy(), cache_o[k]) <= TOL, k
    res = gpu_step(sh, c.q[1], c.q[0], c.K, c.V, meta, c.kb[1], c.vb[1],
                   cache_g["o_p"].clone(), cache_g["l_p"].clone())
    check_step_full(c, 1, res, cache_o, kmin, kmax, tag=f"grown {dtype}")
    assert api.read_device_status(res["ws"]) == api.LOSA_OK
