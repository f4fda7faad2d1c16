"""Full-size parity on the Wan-like, HunyuanVideo-like and sweep workloads.

Same call sequence as bench.py's explicit path (reorder -> mask -> attention
-> unreorder), and the bench's default path in its own test.  The mask is
compared with the oracle on every row of every head, with the near-threshold
exemption.  Attention is compared on seeded query blocks in every head (plus
the first and the last block); the oracle always runs on its own mask.  The
GPU's output on its own mask is compared on the blocks whose mask rows equal
the oracle's, and the GPU's output on the oracle's mask (expanded to lists on
the GPU) on every sampled block.
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

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def built():
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    dbst.load()
    return True


def run_path(w, p, sta, q, k, v):
    """The bench's call sequence on device; returns tiled/raster outputs and the GPU mask."""
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    qd, kd, vd = (P.bits_to_torch(a) for a in (q, k, v))
    qt, kt, vt = (dbst.tile_reorder(x, g) for x in (qd, kd, vd))
    bits, cnt, idx = dbst.build_block_mask(qt, kt, g, p, sta)
    ot, lse = dbst.block_sparse_attn(qt, kt, vt, g, cnt, idx)
    o = dbst.tile_unreorder(ot, g)
    dbst.get_error()
    return g, (qt, kt, vt), bits, cnt, idx, ot, lse, o


def check_full(name, p, per_head=8):
    w = S.workload(name)
    og = P.geometry(w)
    q, k, v = S.make_qkv(w)
    g, dev_t, bits, cnt, idx, ot, lse, o = run_path(w, p, w.sta_radius, q, k, v)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    # reorder and unreorder, bit-exact
    np.testing.assert_array_equal(P.torch_to_bits(dev_t[0]), qt)
    np.testing.assert_array_equal(O.tile_unreorder(P.torch_to_bits(ot), og), P.torch_to_bits(o))
    # mask on every row, near-threshold exemption
    ref, A = P.oracle_mask_per_head(qt, kt, og, p, w.sta_radius)
    got = P.unpack_mask(bits.cpu().numpy().view(np.uint32), og.NB)
    hard, excused = P.mask_mismatches(got, ref, A, p, O.sta_mask(og, w.sta_radius))
    P.write_mask_report(name, p, hard, excused, A)
    ties = sum(P.near_tie(A, p, *t) for t in hard)
    assert not hard, f"{len(hard)} non-excused mask disagreements ({ties} at a near-tie), first {hard[:5]}"
    cnt_h, idx_h = cnt.cpu().numpy(), idx.cpu().numpy()
    assert np.array_equal(cnt_h, got.sum(-1))
    # attention on sampled query blocks computed on the GPU's own lists, against the oracle on its
    # own mask, where the two masks' rows agree (everywhere but at excused near-threshold blocks)
    scale = 1.0 / math.sqrt(w.D)
    rows = P.sample_rows_per_head(w.B, w.H, og.NB, per_head, seed=7 + w.index)
    for (b, h, i) in rows:
        js = idx_h[b, h, i, :cnt_h[b, h, i]]
        assert np.array_equal(js, np.nonzero(got[b, h, i])[0])
    same = P.rows_where_masks_agree(got, ref, rows)
    assert len(same) >= 0.9 * len(rows)
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, ref, 64, scale, rows=same)
    o_gpu = P.gpu_rows(ot, same)
    max_abs, rel = P.attn_errors(o_gpu, o_ref)
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    lse_gpu = np.stack([lse[b, h, i * 64:(i + 1) * 64].cpu().numpy() for (b, h, i) in same]).astype(np.float64)
    assert np.max(np.abs(lse_gpu - lse_ref)) <= P.LSE_MAX_ABS
    # given the oracle's own mask, the same rows again
    words = torch.from_numpy(P.pack_mask(ref).view(np.int32)).cuda()
    rc, ri = dbst.mask_from_bits(words, g)
    ot2, _ = dbst.block_sparse_attn(*dev_t, g, rc, ri)
    dbst.get_error()
    o_ref2, _ = O.masked_attention(qt, kt, vt, ref, 64, scale, rows=rows)
    max_abs2, rel2 = P.attn_errors(P.gpu_rows(ot2, rows), o_ref2)
    assert max_abs2 <= P.ATTN_MAX_ABS and rel2 <= P.ATTN_REL_L2, (max_abs2, rel2)
    return float(ref.mean()), len(excused)


def test_wan_like_full_size(built):
    kept, excused = check_full("wan", 0.9, per_head=16)
    assert 0.05 < kept < 0.15


def test_wan_like_full_size_bench_path(built):
    """The benchmarked configuration: raster q, k, v in, the pair list, raster o and lse out."""
    w = S.workload("wan")
    og = P.geometry(w)
    q, k, v = S.make_qkv(w)
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    qd, kd, vd = (P.bits_to_torch(a) for a in (q, k, v))
    bits, cnt, idx = dbst.build_block_mask_raster(qd, kd, g, 0.9, w.sta_radius)
    pairs = dbst.pair_query_blocks(bits, g)
    o, lse = dbst.block_sparse_attn_raster(qd, kd, vd, g, cnt, idx, pairs=pairs)
    dbst.get_error()
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    ref, A = P.oracle_mask_per_head(qt, kt, og, 0.9, w.sta_radius)
    got = P.unpack_mask(bits.cpu().numpy().view(np.uint32), og.NB)
    hard, _ = P.mask_mismatches(got, ref, A, 0.9, O.sta_mask(og, w.sta_radius))
    assert not hard, f"{len(hard)} non-excused mask disagreements, first {hard[:5]}"
    assert P.lists_match_bits(cnt.cpu().numpy(), idx.cpu().numpy(), got)
    e = pairs.cpu().numpy().astype(np.int64)
    qa, qb = e & 0xFFFF, (e >> 16) & 0xFFFF
    for h in range(og.H):
        seen = np.bincount(np.concatenate([qa[0, h], qb[0, h][qb[0, h] != 0xFFFF]]), minlength=og.NB)
        assert (seen == 1).all()
    # sampled query blocks where the GPU's mask rows equal the oracle's, the oracle on its own mask
    scale = 1.0 / math.sqrt(w.D)
    rows = P.rows_where_masks_agree(got, ref, P.sample_rows_per_head(w.B, w.H, og.NB, 16, seed=17))
    assert len(rows) >= 0.9 * 16 * w.B * w.H
    o_ref_t, lse_ref_t = O.masked_attention(qt, kt, vt, ref, 64, scale, rows=rows)
    o_t = dbst.tile_reorder(o, g)                       # back to tile order to pick the sampled blocks
    lse_t = O.tile_reorder(lse.cpu().numpy()[..., None], og)[..., 0]
    max_abs, rel = P.attn_errors(P.gpu_rows(o_t, rows), o_ref_t)
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    lse_gpu = np.stack([lse_t[b, h, i * 64:(i + 1) * 64] for (b, h, i) in rows]).astype(np.float64)
    assert np.max(np.abs(lse_gpu - lse_ref_t)) <= P.LSE_MAX_ABS


def test_wan_like_2x4x8_variant_full_size(built):
    """The Wan-like latent in 2x4x8 tiles on the grid padded to 22 frames (616 blocks)."""
    kept, excused = check_full("wan_2x4x8", 0.9, per_head=8)
    assert 0.05 < kept < 0.15


def test_hunyuan_like_full_size(built):
    kept, excused = check_full("hunyuan", 0.9, per_head=64)
    assert 0.03 < kept < 0.15


# every p of the sparsity sweep
@pytest.mark.parametrize("p", S.workload("sweep").p_list)
def test_sweep_full_size(built, p):
    kept, excused = check_full("sweep", p, per_head=8)
    if p >= 1.0:
        assert kept == 1.0


def test_sweep_dense_equals_p1(built):
    w = S.workload("sweep")
    q, k, v = S.make_qkv(w, heads=range(2), batches=range(1))
    w2 = dataclasses.replace(w, B=1, H=2)
    g = dbst.Geom.make(1, 2, w.D, w.grid, w.tile)
    qt, kt, vt = (dbst.tile_reorder(P.bits_to_torch(a), g) for a in (q, k, v))
    bits, cnt, idx = dbst.build_block_mask(qt, kt, g, 1.0, -1)
    o1, l1 = dbst.block_sparse_attn(qt, kt, vt, g, cnt, idx)
    o2, l2 = dbst.dense_attn(qt, kt, vt, g)
    dbst.get_error()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    del w2
