"""Full-size parity of the attention backward on the Wan-like workload.

The launch configuration is the one ``bench.py --backward`` times: raster
layout, all 40 heads, p = 0.9.  The GPU runs on the oracle's own mask (packed,
expanded and transposed on the GPU), so every oracle input is the oracle's.
The oracle computes dq for seeded query blocks in every head plus the first
and the last block, and dk, dv for seeded key blocks in every fifth head plus
the first and the last; each dk/dv block needs every query row that keeps it.
Bounds as in test_gpu_backward.py.
"""
import math

import numpy as np
import pytest
import torch

import dbst_synth as S
import oracle as O
import dynamic_block_sparse_tile_b200 as dbst
from tests import parity as P
from tests.test_gpu_backward import GRAD_MAX_REL, GRAD_REL_L2

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def built():
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    dbst.load()
    return True


def sample_blocks(H, NB, seed=2024):
    rng = np.random.default_rng(seed)
    qs = [(0, h, int(i)) for h in range(H) for i in rng.choice(NB, 2, replace=False)]
    ks = [(0, h, int(rng.integers(NB))) for h in range(0, H, 5)]
    return qs + [(0, 0, 0), (0, H - 1, NB - 1)], ks + [(0, 0, 0), (0, H - 1, NB - 1)]


def compare(name, got, ref):
    got, ref = np.concatenate(got), np.concatenate(ref)
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err.max() <= GRAD_MAX_REL * np.abs(ref).max(), (name, err.max(), np.abs(ref).max())
    assert rel <= GRAD_REL_L2, (name, rel)


def test_wan_like_backward_full_size_sampled(built):
    w = S.workload("wan")
    p = w.p_list[0]
    og = P.geometry(w)
    q, k, v = S.make_qkv(w)
    do = S.make_grad(w)
    qt, kt = O.tile_reorder(q, og), O.tile_reorder(k, og)
    mask, _ = P.oracle_mask_per_head(qt, kt, og, p, w.sta_radius)

    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    tq, tk, tv, tdo = (P.bits_to_torch(a) for a in (q, k, v, do))
    bits = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(bits, g)
    _, qcnt, qidx = dbst.transpose_block_mask(bits, g)
    pairs = dbst.pair_query_blocks(bits, g)
    _, lse = dbst.block_sparse_attn_raster(tq, tk, tv, g, cnt, idx, pairs=pairs)
    dq, dk, dv = dbst.block_sparse_attn_backward(tq, tk, tv, lse, tdo, g, cnt, idx, qcnt, qidx, raster=True)
    dbst.get_error()
    dq, dk, dv = (S.f32_from_bf16_bits(O.tile_reorder(P.torch_to_bits(t), og)) for t in (dq, dk, dv))
    del tq, tk, tv, tdo

    qs, ks = sample_blocks(w.H, og.NB)
    vt = O.tile_reorder(v, og)
    dot = S.f32_from_bf16_bits(O.tile_reorder(do, og))
    gq, gkv = O.masked_attention_backward_blocks(qt, kt, vt, mask, 64, 1.0 / math.sqrt(w.D), dot, qs, ks)
    sl = lambda i: slice(64 * i, 64 * i + 64)   # noqa: E731
    compare("dq", [dq[b, h, sl(i)] for b, h, i in qs], [gq[t] for t in qs])
    compare("dk", [dk[b, h, sl(j)] for b, h, j in ks], [gkv[t][0] for t in ks])
    compare("dv", [dv[b, h, sl(j)] for b, h, j in ks], [gkv[t][1] for t in ks])
