"""Raster-order entry points: the tile reorder folded into the kernels' own loads and stores.

Each case runs the path twice on the same raster q, k, v: once through
`dbst_tile_reorder` + the tiled entry points + `dbst_tile_unreorder`, once
through the `_raster` entry points.  The two must agree bit for bit (mask
words, lists, o, lse), and one case is also checked against the oracle.
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


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def _lse_to_raster(lse_tiled, og):
    a = lse_tiled.cpu().numpy()[..., None]
    return O.tile_unreorder(a, og)[..., 0]


def both_paths(w, p, sta, heads=None, batches=None):
    og = P.geometry(w, heads=None if heads is None else len(heads))
    if batches is not None:
        og = dataclasses.replace(og, B=len(batches))
    g = dbst.Geom.make(og.B, og.H, og.D, (og.T, og.Y, og.X), (og.tt, og.ty, og.tx))
    q, k, v = S.make_qkv(w, heads=heads, batches=batches)
    qd, kd, vd = (P.bits_to_torch(a) for a in (q, k, v))
    qt, kt, vt = (dbst.tile_reorder(x, g) for x in (qd, kd, vd))
    tiled = {}
    tiled["mask"] = dbst.build_block_mask(qt, kt, g, p, sta)
    ot, lt = dbst.block_sparse_attn(qt, kt, vt, g, tiled["mask"][1], tiled["mask"][2])
    tiled["o"], tiled["lse"] = dbst.tile_unreorder(ot, g), lt
    od, ld = dbst.dense_attn(qt, kt, vt, g)
    tiled["od"], tiled["lsed"] = dbst.tile_unreorder(od, g), ld
    raster = {}
    raster["mask"] = dbst.build_block_mask_raster(qd, kd, g, p, sta)
    raster["o"], raster["lse"] = dbst.block_sparse_attn_raster(qd, kd, vd, g, raster["mask"][1], raster["mask"][2])
    raster["od"], raster["lsed"] = dbst.dense_attn_raster(qd, kd, vd, g)
    dbst.get_error()
    return og, (q, k, v), tiled, raster


def assert_identical(og, tiled, raster):
    (bt, ct, it), (br, cr, ir) = tiled["mask"], raster["mask"]
    assert torch.equal(bt, br) and torch.equal(ct, cr)
    valid = torch.arange(it.shape[-1], device=it.device) < ct[..., None]   # entries past kv_count are unspecified
    assert torch.equal(it[valid], ir[valid])
    assert torch.equal(_bits(tiled["o"]), _bits(raster["o"]))
    assert torch.equal(_bits(tiled["od"]), _bits(raster["od"]))
    np.testing.assert_array_equal(_lse_to_raster(tiled["lse"], og), raster["lse"].cpu().numpy())
    np.testing.assert_array_equal(_lse_to_raster(tiled["lsed"], og), raster["lsed"].cpu().numpy())


CASES = [("tiny", 0.9, -1), ("small", 0.9, 1), ("small", 0.5, 0), ("small", 1.0, -1)]


@pytest.mark.parametrize("name,p,sta", CASES)
def test_raster_equals_reorder_then_tiled(built, name, p, sta):
    og, _, tiled, raster = both_paths(S.workload(name), p, sta)
    assert_identical(og, tiled, raster)


@pytest.mark.parametrize("D,grid,tile", [(128, (4, 16, 32), (2, 4, 8)), (64, (6, 8, 24), (1, 8, 8)),
                                         (128, (2, 32, 16), (2, 8, 4))])
def test_raster_other_tilings(built, D, grid, tile):
    w = S.Workload("rt", 8, B=2, H=2, D=D, grid=grid, tile=tile, alpha=0.7, beta=0.3, f_rms=2.0, kmax=3,
                   p_list=(0.8,), sta_radius=1)
    og, _, tiled, raster = both_paths(w, 0.8, 1)
    assert_identical(og, tiled, raster)


def test_raster_against_oracle(built):
    w = S.workload("small")
    og, (q, k, v), _, raster = both_paths(w, 0.9, 1)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    got = P.unpack_mask(raster["mask"][0].cpu().numpy().view(np.uint32), og.NB)
    # the oracle on its own mask; outputs compared on the query blocks whose mask rows agree
    ref = O.build_block_mask(qt, kt, og, 0.9, 1)
    agree = (got == ref).all(-1)
    assert agree.mean() >= 0.9
    sel = np.repeat(agree, 64, axis=-1)
    o_ref_t, lse_ref_t = O.masked_attention(qt, kt, vt, ref, 64, 1.0 / math.sqrt(w.D))
    o_t = O.tile_reorder(raster["o"].float().cpu().numpy().astype(np.float64), og)
    lse_t = O.tile_reorder(raster["lse"].cpu().numpy()[..., None], og)[..., 0]
    max_abs, rel = P.attn_errors(o_t[sel], o_ref_t[sel])
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    assert np.max(np.abs(lse_t[sel] - lse_ref_t[sel])) <= P.LSE_MAX_ABS


@pytest.mark.slow
def test_raster_wan_like_full_size(built):
    w = S.workload("wan")
    og, _, tiled, raster = both_paths(w, 0.9, -1, heads=range(0, 40, 5))
    assert_identical(og, tiled, raster)
