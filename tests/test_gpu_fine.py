"""GPU parity of the fine-grained path (AB-Attention page, section "Les trois
techniques", third technique: key groups of 4 tokens) against the float64
oracle ``oracle.fine``.

Selection: the kept groups must match the oracle's, a disagreement being
excused only where the oracle's cumulative pooled mass at that group's rank,
or the rank before it, lies within 1e-4 of p (the rule of the block mask).
Attention over the kept groups, on the oracle's own mask: the forward's bounds.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

import dbst_synth as S
import oracle as O
import dynamic_block_sparse_tile_b200 as dbst
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def built():
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    dbst.load()
    return True


def gpu_geom(w):
    return dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)


def groups_from_masks(gm: np.ndarray) -> np.ndarray:
    """int16 [B, H, NB, NB] group masks -> bool [B, H, NB, 16 * NB] kept groups."""
    u = gm.view(np.uint16).astype(np.uint32)
    bits = (u[..., None] >> np.arange(16, dtype=np.uint32)) & 1
    return bits.reshape(*gm.shape[:-1], gm.shape[-1] * 16).astype(bool)


def masks_from_groups(keep: np.ndarray) -> np.ndarray:
    """bool [B, H, NB, 16 * NB] -> int16 group masks [B, H, NB, NB]."""
    b = keep.reshape(*keep.shape[:-1], -1, 16).astype(np.uint32)
    return (b << np.arange(16, dtype=np.uint32)).sum(-1).astype(np.uint16).view(np.int16)


def hard_mismatches(got, ref, A, p):
    bad = []
    for b, h, i, j in np.argwhere(got != ref):
        a = A[b, h, i]
        order = np.argsort(-a, kind="stable")
        c = np.cumsum(a[order])
        rank = int(np.nonzero(order == j)[0][0])
        near = abs(c[rank] - p) <= P.CDF_EXEMPT or (rank > 0 and abs(c[rank - 1] - p) <= P.CDF_EXEMPT)
        if not near or p >= 1.0:
            bad.append((int(b), int(h), int(i), int(j)))
    return bad


@pytest.mark.parametrize("name,p,D", [("tiny", 0.9, 64), ("tiny", 1.0, 64), ("small", 0.9, 64),
                                      ("small", 0.7, 128)])
def test_fine_mask_matches_oracle(built, name, p, D):
    w = dataclasses.replace(S.workload(name), D=D)
    og = P.geometry(w)
    g = gpu_geom(w)
    q, k, _ = S.make_qkv(w)
    qt, kt = (O.tile_reorder(a, og) for a in (q, k))
    gm, cnt, idx = dbst.build_fine_mask(P.bits_to_torch(qt), P.bits_to_torch(kt), g, p)
    dbst.get_error()
    got = groups_from_masks(gm.cpu().numpy())
    ref, A = O.build_fine_mask(qt, kt, og, p, G=4, return_scores=True)
    assert not hard_mismatches(got, ref, A, p)
    blocks = got.reshape(*got.shape[:-1], og.NB, 16).any(-1)
    assert P.lists_match_bits(cnt.cpu().numpy(), idx.cpu().numpy(), blocks)
    # the fused form reads raster q, k and gives the same bits
    gm_r, cnt_r, idx_r = dbst.build_fine_mask(P.bits_to_torch(q), P.bits_to_torch(k), g, p, raster=True)
    dbst.get_error()
    assert torch.equal(gm, gm_r) and torch.equal(cnt, cnt_r)


@pytest.mark.parametrize("name,p,D", [("tiny", 0.9, 64), ("small", 0.9, 64), ("small", 0.7, 128)])
def test_group_attention_matches_oracle(built, name, p, D):
    w = dataclasses.replace(S.workload(name), D=D)
    og = P.geometry(w)
    g = gpu_geom(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    keep = O.build_fine_mask(qt, kt, og, p, G=4)
    keep[0, 0, 1] = False                                     # an empty row
    gm = torch.from_numpy(masks_from_groups(keep)).cuda()
    blocks = keep.reshape(*keep.shape[:-1], og.NB, 16).any(-1)
    cnt, idx = dbst.mask_from_bits(torch.from_numpy(P.pack_mask(blocks).view(np.int32)).cuda(), g)
    o, lse = dbst.block_sparse_attn_groups(*(P.bits_to_torch(a) for a in (qt, kt, vt)), g, cnt, idx, gm)
    dbst.get_error()
    ref_o, ref_lse = O.fine_masked_attention(qt, kt, vt, keep, 64, 4, 1.0 / math.sqrt(D))
    got = S.f32_from_bf16_bits(P.torch_to_bits(o)).astype(np.float64)
    max_abs, rel = P.attn_errors(got, ref_o)
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    lse = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert (np.isneginf(lse) == ~fin).all()
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= P.LSE_MAX_ABS
    # raster layout: the same bits
    ro, rlse = dbst.block_sparse_attn_groups(*(P.bits_to_torch(a) for a in (q, k, v)), g, cnt, idx, gm, raster=True)
    dbst.get_error()
    np.testing.assert_array_equal(O.tile_reorder(P.torch_to_bits(ro), og), P.torch_to_bits(o))


@pytest.mark.parametrize("name,p,D", [("tiny", 0.9, 64), ("small", 0.9, 64), ("small", 0.7, 128)])
def test_gathered_group_attention_matches_oracle(built, name, p, D):
    """The page's design: kept groups gathered 16 to a 64-key tile by 4-row loads."""
    w = dataclasses.replace(S.workload(name), D=D)
    og = P.geometry(w)
    g = gpu_geom(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    keep = O.build_fine_mask(qt, kt, og, p, G=4)
    keep[0, 0, 1] = False                                     # an empty row
    gm = torch.from_numpy(masks_from_groups(keep)).cuda()
    o, lse = dbst.block_sparse_attn_gather(*(P.bits_to_torch(a) for a in (qt, kt, vt)), g, gm)
    dbst.get_error()
    ref_o, ref_lse = O.fine_masked_attention(qt, kt, vt, keep, 64, 4, 1.0 / math.sqrt(D))
    got = S.f32_from_bf16_bits(P.torch_to_bits(o)).astype(np.float64)
    max_abs, rel = P.attn_errors(got, ref_o)
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    lse = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert (np.isneginf(lse) == ~fin).all()
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= P.LSE_MAX_ABS
    ro, _ = dbst.block_sparse_attn_gather(*(P.bits_to_torch(a) for a in (q, k, v)), g, gm, raster=True)
    dbst.get_error()
    np.testing.assert_array_equal(O.tile_reorder(P.torch_to_bits(ro), og), P.torch_to_bits(o))
