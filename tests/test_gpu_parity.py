"""GPU parity: every step of the path, through the C ABI, against the oracle.

Small workloads (tiny, small) are compared element by element on every
output.  Edge cases use caller-supplied masks (empty rows, single blocks, odd
counts, all ones).  Full-size workloads live in test_gpu_fullsize.py.
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


def gpu_geom(w, heads=None):
    return dbst.Geom.make(w.B, w.H if heads is None else heads, w.D, w.grid, w.tile)


@pytest.fixture(scope="module")
def built():
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    dbst.load()
    return True


def run_reorder(w, q):
    g = gpu_geom(w)
    x = P.bits_to_torch(q)
    y = dbst.tile_reorder(x, g)
    z = dbst.tile_unreorder(y, g)
    dbst.get_error()
    return P.torch_to_bits(y), P.torch_to_bits(z)


# ---------------------------------------------------------------- reorder
@pytest.mark.parametrize("name", ["tiny", "small", "sweep"])
def test_reorder_is_bit_exact(built, name):
    w = S.workload(name)
    q, _, _ = S.make_qkv(w, heads=range(min(w.H, 4)))
    w4 = dataclasses.replace(w, H=q.shape[1])
    y, z = run_reorder(w4, q)
    np.testing.assert_array_equal(y, O.tile_reorder(q, P.geometry(w4)))
    np.testing.assert_array_equal(z, q)


@pytest.mark.parametrize("grid,tile", [((4, 8, 16), (2, 4, 8)), ((2, 16, 8), (2, 4, 8)), ((3, 8, 24), (1, 8, 8)),
                                       ((4, 4, 16), (4, 4, 4)), ((1, 64, 8), (1, 8, 8))])
@pytest.mark.parametrize("D", [64, 128])
def test_reorder_other_tilings(built, grid, tile, D):
    w = S.Workload("t", 0, B=2, H=3, D=D, grid=grid, tile=tile, alpha=0.7, beta=0.3, f_rms=1.0, kmax=1,
                   p_list=(0.9,), sta_radius=-1)
    q, _, _ = S.make_qkv(w)
    y, z = run_reorder(w, q)
    np.testing.assert_array_equal(y, O.tile_reorder(q, P.geometry(w)))
    np.testing.assert_array_equal(z, q)


# ---------------------------------------------------------------- mask
def gpu_mask(w, qt_bits, kt_bits, p, sta, heads=None):
    g = gpu_geom(w, heads)
    bits, cnt, idx = dbst.build_block_mask(P.bits_to_torch(qt_bits), P.bits_to_torch(kt_bits), g, p, sta)
    dbst.get_error()
    bits = bits.cpu().numpy().view(np.uint32)
    return P.unpack_mask(bits, g.NB), cnt.cpu().numpy(), idx.cpu().numpy()


MASK_CASES = [("tiny", 0.9, -1), ("tiny", 1.0, -1), ("small", 0.8, 1), ("small", 0.9, 1), ("small", 0.95, 1),
              ("small", 0.9, -1), ("small", 0.5, 0), ("small", 1.0, 2)]


@pytest.mark.parametrize("name,p,sta", MASK_CASES)
def test_mask_matches_oracle(built, name, p, sta):
    w = S.workload(name)
    g = P.geometry(w)
    q, k, _ = S.make_qkv(w)
    qt, kt = O.tile_reorder(q, g), O.tile_reorder(k, g)
    ref, A = P.oracle_mask_per_head(qt, kt, g, p, sta)
    got, cnt, idx = gpu_mask(w, qt, kt, p, sta)
    hard, excused = P.mask_mismatches(got, ref, A, p, O.sta_mask(g, sta))
    assert not hard, f"{len(hard)} non-excused mask disagreements, first {hard[:5]}"
    assert P.lists_match_bits(cnt, idx, got)
    assert (cnt >= 1).all()
    if p >= 1.0:
        assert got.all()


# Rows of more than 1024 blocks (the HunyuanVideo-like shape has 2040): the tensor-core path's longest
# rows, with integer masses in coarser units, and beyond 2048 blocks the float64 path; the whole mask
# against the oracle.
@pytest.mark.parametrize("grid,p,sta", [((17, 64, 64), 0.9, -1), ((32, 64, 64), 0.8, 1), ((34, 64, 64), 0.9, -1)])
def test_mask_long_rows_match_oracle(built, grid, p, sta):
    w = dataclasses.replace(S.workload("small"), H=2, grid=grid, tile=(1, 8, 8))
    g = P.geometry(w)
    assert 1024 < g.NB <= 4096
    q, k, _ = S.make_qkv(w)
    qt, kt = O.tile_reorder(q, g), O.tile_reorder(k, g)
    ref, A = P.oracle_mask_per_head(qt, kt, g, p, sta)
    got, cnt, idx = gpu_mask(w, qt, kt, p, sta)
    hard, excused = P.mask_mismatches(got, ref, A, p, O.sta_mask(g, sta))
    assert not hard, f"{len(hard)} non-excused mask disagreements, first {hard[:5]}"
    assert P.lists_match_bits(cnt, idx, got)


# ---------------------------------------------------------------- attention
def gpu_attention_from_mask(w, qt, kt, vt, mask, scale=0.0):
    g = gpu_geom(w, heads=qt.shape[1])
    words = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(words, g)
    o, lse = dbst.block_sparse_attn(P.bits_to_torch(qt), P.bits_to_torch(kt), P.bits_to_torch(vt), g, cnt, idx,
                                    scale)
    dbst.get_error()
    assert P.lists_match_bits(cnt.cpu().numpy(), idx.cpu().numpy(), mask)
    return o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64)


def check_attention(o, lse, o_ref, lse_ref):
    max_abs, rel = P.attn_errors(o, o_ref)
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    fin = np.isfinite(lse_ref)
    np.testing.assert_array_equal(np.isfinite(lse), fin)
    assert (np.isneginf(lse[~fin])).all()
    if fin.any():
        assert np.max(np.abs(lse[fin] - lse_ref[fin])) <= P.LSE_MAX_ABS


@pytest.mark.parametrize("name,p,sta", [("tiny", 0.9, -1), ("tiny", 1.0, -1), ("small", 0.8, 1),
                                        ("small", 0.95, 1), ("small", 0.9, -1)])
def test_attention_with_oracle_mask(built, name, p, sta):
    w = S.workload(name)
    g = P.geometry(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
    mask = O.build_block_mask(qt, kt, g, p, sta)
    scale = 1.0 / math.sqrt(w.D)
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, mask, 64, scale)
    o, lse = gpu_attention_from_mask(w, qt, kt, vt, mask)
    check_attention(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("name", ["tiny", "small"])
def test_dense_attention(built, name):
    w = S.workload(name)
    g = P.geometry(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
    o_ref, lse_ref = O.dense_attention(qt, kt, vt, 1.0 / math.sqrt(w.D))
    o, lse = dbst.dense_attn(P.bits_to_torch(qt), P.bits_to_torch(kt), P.bits_to_torch(vt), gpu_geom(w))
    dbst.get_error()
    check_attention(o.float().cpu().numpy().astype(np.float64), lse.cpu().numpy().astype(np.float64),
                    o_ref, lse_ref)


def edge_masks(NB, seed):
    rng = np.random.default_rng(seed)
    m = rng.random((NB, NB)) < 0.35
    m[0] = False                           # empty row
    m[1] = False
    m[1, NB - 1] = True                    # single (last) block
    m[2] = False
    m[2, [0, 3, 5]] = True                 # odd count
    m[3] = True                            # all blocks
    if NB > 8:
        m[4] = False
        m[4, 4] = True                     # single diagonal block
    return m


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("NBgrid", [((4, 16, 16), (1, 8, 8)), ((2, 8, 64), (1, 8, 8))])
def test_attention_edge_masks(built, D, NBgrid):
    grid, tile = NBgrid
    w = S.Workload("edge", 5, B=1, H=2, D=D, grid=grid, tile=tile, alpha=0.7, beta=0.3, f_rms=2.0, kmax=3,
                   p_list=(0.9,), sta_radius=-1)
    g = P.geometry(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
    mask = np.stack([edge_masks(g.NB, s) for s in range(w.H)])[None]
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, mask, 64, 0.11)
    o, lse = gpu_attention_from_mask(w, qt, kt, vt, mask, scale=0.11)
    check_attention(o, lse, o_ref, lse_ref)
    assert (o[0, 0, :64] == 0).all() and np.isneginf(lse[0, 0, :64]).all()


def test_attention_repeat_launches_bit_identical(built):
    """Repeated launches on the same inputs give bit-identical outputs.

    The kernel's warps hand tiles to one another through barriers; an ordering
    bug between them shows up as run-to-run differences long before it shows
    up as a tolerance failure on one run.
    """
    w = S.Workload("rep", 7, B=1, H=4, D=128, grid=(4, 16, 32), tile=(1, 8, 8), alpha=0.7, beta=0.3, f_rms=4.0,
                   kmax=3, p_list=(0.9,), sta_radius=-1)
    g = P.geometry(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
    mask = np.stack([edge_masks(g.NB, s) for s in range(w.H)])[None]
    gg = gpu_geom(w, heads=w.H)
    words = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(words, gg)
    qd, kd, vd = (P.bits_to_torch(a) for a in (qt, kt, vt))
    o0, l0 = dbst.block_sparse_attn(qd, kd, vd, gg, cnt, idx, 0.3)
    for _ in range(30):
        o1, l1 = dbst.block_sparse_attn(qd, kd, vd, gg, cnt, idx, 0.3)
        assert torch.equal(o0.view(torch.int16), o1.view(torch.int16))
        assert torch.equal(l0, l1)
    dbst.get_error()
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, mask, 64, 0.3)
    check_attention(o0.float().cpu().numpy().astype(np.float64), l0.cpu().numpy().astype(np.float64), o_ref, lse_ref)


@pytest.mark.parametrize("raster", [False, True])
def test_heads_with_no_kept_blocks(built, raster):
    """Every pair of query blocks empty in one head (the kernel's early exit), full lists in the other."""
    w = S.Workload("empty", 9, B=1, H=2, D=128, grid=(4, 16, 32), tile=(1, 8, 8), alpha=0.7, beta=0.3, f_rms=2.0,
                   kmax=3, p_list=(0.9,), sta_radius=-1)
    g = P.geometry(w)
    q, k, v = S.make_qkv(w)
    mask = np.zeros((1, 2, g.NB, g.NB), bool)
    mask[0, 1] = True
    gg = gpu_geom(w)
    words = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(words, gg)
    if raster:
        o, lse = dbst.block_sparse_attn_raster(*(P.bits_to_torch(a) for a in (q, k, v)), gg, cnt, idx)
        o = dbst.tile_reorder(o, gg)
        lse = torch.from_numpy(O.tile_reorder(lse.cpu().numpy()[..., None], g)[..., 0])
    else:
        qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
        o, lse = dbst.block_sparse_attn(*(P.bits_to_torch(a) for a in (qt, kt, vt)), gg, cnt, idx)
    dbst.get_error()
    o = o.float().cpu().numpy()
    lse = lse.cpu().numpy()
    assert (o[0, 0] == 0).all() and np.isneginf(lse[0, 0]).all()
    qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, mask, 64, 1.0 / math.sqrt(w.D))
    check_attention(o.astype(np.float64), lse.astype(np.float64), o_ref, lse_ref)


def test_constant_v_and_large_logits(built):
    """Constant V is reproduced; logits spanning > 2^16 in log2 units force rescales."""
    w = S.Workload("c", 6, B=1, H=1, D=128, grid=(2, 16, 32), tile=(2, 4, 8), alpha=0.7, beta=0.3, f_rms=6.0,
                   kmax=3, p_list=(0.9,), sta_radius=-1)
    g = P.geometry(w)
    q, k, _ = S.make_qkv(w)
    qt, kt = (O.tile_reorder(a, g) for a in (q, k))
    const = S.bf16_bits_from_f32(np.linspace(-2, 2, 128, dtype=np.float32))
    vt = np.broadcast_to(const, qt.shape).copy()
    mask = np.ones((1, 1, g.NB, g.NB), bool)
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, mask, 64, 0.5)
    o, lse = gpu_attention_from_mask(w, qt, kt, vt, mask, scale=0.5)
    check_attention(o, lse, o_ref, lse_ref)


def test_out_of_range_list_entries_are_reported(built):
    w = S.workload("tiny")
    g = gpu_geom(w)
    q, k, v = (P.bits_to_torch(a) for a in S.make_qkv(w))
    cnt = torch.full((1, 2, 4), 2, dtype=torch.int32, device="cuda")
    idx = torch.zeros((1, 2, 4, 4), dtype=torch.int16, device="cuda")
    idx[..., 1] = 7                                   # NB = 4: entry 7 is out of range
    dbst.block_sparse_attn(q, k, v, g, cnt, idx)
    with pytest.raises(dbst.DbstError) as e:
        dbst.get_error()
    assert e.value.status == dbst.DBST_EBOUNDS
    dbst.get_error()                                  # cleared after reporting
