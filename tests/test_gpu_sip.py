"""GPU parity of SIP (AB-Attention page, section "Les trois techniques": sampled
key blocks weighted by the inverse inclusion probability) against the float64
oracle.

Selection: the kept set is compared block by block with the oracle's (same
uniforms, drawn here from a seeded generator and given to both sides); a
disagreement is excused only where the uniform lies within 1e-9 of the
oracle's pi (the two sides sum the pooled map in different orders, so pi agrees
to about 1e-15).  Offsets log(1/pi) agree to float32 rounding.

Attention with offsets: the forward kernel, offsets in its exponent, against ``oracle.sip_attention``
on the oracle's own kept set and pi, with the forward's bounds (max-abs 2e-2,
relative L2 5e-3 on o, 2e-3 on lse); without offsets it must match the plain
masked attention oracle to the same bounds.
"""
import dataclasses

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


def oracle_pi(w, q, k, budget):
    og = P.geometry(w)
    qt, kt = (O.bf16_bits_to_f64(O.tile_reorder(a, og)) for a in (q, k))
    A = O.pooled_score_map(O.block_mean_pool(qt, 64), O.block_mean_pool(kt, 64), 1.0 / np.sqrt(w.D))
    return O.inclusion_probabilities(A, budget)


def check_attention(name, o, lse, ref_o, ref_lse):
    got = S.f32_from_bf16_bits(P.torch_to_bits(o)).astype(np.float64)
    err = np.abs(got - ref_o)
    assert err.max() <= P.ATTN_MAX_ABS, (name, err.max())
    nz = np.linalg.norm(ref_o)
    if nz > 0:
        assert np.linalg.norm(got - ref_o) / nz <= P.ATTN_REL_L2, name
    lse = lse.cpu().numpy()
    fin = np.isfinite(ref_lse)
    assert (np.isneginf(lse) == ~fin).all(), name
    assert np.abs(lse[fin] - ref_lse[fin]).max() <= P.LSE_MAX_ABS, name


@pytest.mark.parametrize("name,budget", [("tiny", 1.5), ("small", 4.0), ("small", 10.0), ("small", 40.0)])
def test_sip_mask_matches_oracle(built, name, budget):
    w = S.workload(name)
    og = P.geometry(w)
    g = gpu_geom(w)
    q, k, _ = S.make_qkv(w)
    u = np.random.default_rng(31).random((w.B, w.H, og.NB, og.NB))
    qt, kt = (P.bits_to_torch(O.tile_reorder(a, og)) for a in (q, k))
    bits, cnt, idx, off = dbst.build_sip_mask(qt, kt, g, budget, torch.from_numpy(u).cuda())
    dbst.get_error()
    pi = oracle_pi(w, q, k, budget)
    keep = O.sip_sample(pi, u)
    got = P.unpack_mask(bits.cpu().numpy().view(np.uint32), og.NB)
    bad = (got != keep) & ~(np.abs(u - pi) < 1e-9)
    assert not bad.any(), np.argwhere(bad)[:5]
    off = off.cpu().numpy()
    both = got & keep
    np.testing.assert_allclose(off[both], -np.log(pi[both]), rtol=2e-7, atol=2e-7)
    assert (off[~got] == 0).all()
    cnt = cnt.cpu().numpy()
    idx = idx.cpu().numpy()
    np.testing.assert_array_equal(cnt, got.sum(-1))
    for r in np.ndindex(cnt.shape):
        np.testing.assert_array_equal(idx[r][:cnt[r]], np.nonzero(got[r])[0])


def test_sip_mask_raster_equals_tiled(built):
    w = S.workload("small")
    og = P.geometry(w)
    g = gpu_geom(w)
    q, k, _ = S.make_qkv(w)
    u = torch.from_numpy(np.random.default_rng(5).random((w.B, w.H, og.NB, og.NB))).cuda()
    tiled = dbst.build_sip_mask(*(P.bits_to_torch(O.tile_reorder(a, og)) for a in (q, k)), g, 6.0, u)
    raster = dbst.build_sip_mask(P.bits_to_torch(q), P.bits_to_torch(k), g, 6.0, u, raster=True)
    dbst.get_error()
    (bt, ct, it, ot), (br, cr, ir, orr) = tiled, raster
    assert torch.equal(bt, br) and torch.equal(ct, cr) and torch.equal(ot, orr)
    # kv_idx is defined only up to each row's kv_count; the rest of a row is left untouched
    valid = torch.arange(og.NB, device=ct.device) < ct[..., None]
    assert torch.equal(it[valid], ir[valid])


def run_offset_attn(w, q, k, v, keep, off, raster=False):
    g = gpu_geom(w)
    og = P.geometry(w)
    bits = torch.from_numpy(P.pack_mask(keep).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(bits, g)
    offsets = None if off is None else torch.from_numpy(off.astype(np.float32)).cuda()
    if raster:
        o, lse = dbst.block_sparse_attn_offsets(*(P.bits_to_torch(a) for a in (q, k, v)), g, cnt, idx, offsets,
                                                raster=True)
        dbst.get_error()
        return (torch.from_numpy(O.tile_reorder(P.torch_to_bits(o), og).view(np.int16)).view(torch.bfloat16),
                torch.from_numpy(O.tile_reorder(lse.cpu().numpy()[..., None], og)[..., 0]))
    o, lse = dbst.block_sparse_attn_offsets(*(P.bits_to_torch(O.tile_reorder(a, og)) for a in (q, k, v)), g, cnt,
                                            idx, offsets)
    dbst.get_error()
    return o, lse


@pytest.mark.parametrize("name,D", [("tiny", 64), ("small", 64), ("small", 128)])
def test_offset_free_attention_matches_masked_attention(built, name, D):
    w = dataclasses.replace(S.workload(name), D=D)
    og = P.geometry(w)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    mask = O.build_block_mask(qt, kt, og, 0.9, w.sta_radius)
    mask[0, 0, 1] = False                                      # an empty row
    o, lse = run_offset_attn(w, q, k, v, mask, None)
    ref_o, ref_lse = O.masked_attention(qt, kt, vt, mask, 64, 1.0 / np.sqrt(D))
    check_attention(f"{name} D={D}", o, lse, ref_o, ref_lse)


@pytest.mark.parametrize("name,budget,D", [("tiny", 2.0, 64), ("small", 5.0, 64), ("small", 12.0, 128)])
def test_sip_attention_matches_oracle(built, name, budget, D):
    w = dataclasses.replace(S.workload(name), D=D)
    og = P.geometry(w)
    q, k, v = S.make_qkv(w)
    u = np.random.default_rng(17).random((w.B, w.H, og.NB, og.NB))
    pi = oracle_pi(w, q, k, budget)
    keep = O.sip_sample(pi, u)
    off = np.where(keep, -np.log(np.where(keep, pi, 1.0)), 0.0)
    o, lse = run_offset_attn(w, q, k, v, keep, off)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    ref_o, ref_lse = O.sip_attention(qt, kt, vt, keep, pi, 64, 1.0 / np.sqrt(D))
    check_attention(f"{name} K={budget} D={D}", o, lse, ref_o, ref_lse)
    # raster layout: the same bits
    ro, rlse = run_offset_attn(w, q, k, v, keep, off, raster=True)
    assert torch.equal(ro.view(torch.int16), o.view(torch.int16).cpu())
    np.testing.assert_array_equal(rlse.numpy(), lse.cpu().numpy())
    # on the pair schedule of the sampled mask: the same bounds
    g = gpu_geom(w)
    bits = torch.from_numpy(P.pack_mask(keep).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(bits, g)
    pairs = dbst.pair_query_blocks(bits, g)
    po, plse = dbst.block_sparse_attn_offsets(*(P.bits_to_torch(a) for a in (qt, kt, vt)), g, cnt, idx,
                                              torch.from_numpy(off.astype(np.float32)).cuda(), pairs=pairs)
    dbst.get_error()
    check_attention(f"{name} K={budget} D={D} paired", po, plse, ref_o, ref_lse)


def test_offset_attention_empty_head_and_repeat(built):
    w = S.workload("tiny")
    og = P.geometry(w)
    q, k, v = S.make_qkv(w)
    keep = np.ones((w.B, w.H, og.NB, og.NB), bool)
    keep[0, 1] = False
    off = np.full(keep.shape, 0.7)
    a = run_offset_attn(w, q, k, v, keep, off)
    b = run_offset_attn(w, q, k, v, keep, off)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])
    assert not P.torch_to_bits(a[0])[0, 1].any() and np.isneginf(a[1].cpu().numpy()[0, 1]).all()
    # a constant offset on every kept block changes nothing but lse
    ref_o, ref_lse = O.masked_attention(*(O.tile_reorder(x, og) for x in (q, k, v)), keep, 64, 1.0 / 8)
    check_attention("constant offset", a[0], a[1] - 0.7, ref_o, ref_lse)
