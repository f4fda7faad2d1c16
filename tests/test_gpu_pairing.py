"""Query-block pairing (`dbst_pair_query_blocks`) and attention that runs on it.

The pairing is a schedule only: every block of a head must appear exactly once,
and attention on it must agree with the oracle like attention on the fixed
neighbour pairs.  On the seeded content-adaptive masks it must also cost no more
tensor-core tiles than the fixed pairs (it is chosen to cost fewer).
"""
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


def decode(pairs):
    e = pairs.cpu().numpy().astype(np.int64)
    return e & 0xFFFF, (e >> 16) & 0xFFFF


def fixed_pairs(og):
    nT, nY, nX = og.tile_grid
    ps = nY * nX if nT > 1 else (nX if nY > 1 else 1)
    out = []
    for qa in range(og.NB):
        if (qa // ps) % 2 == 0:
            out.append((qa, qa + ps if qa + ps < og.NB else None))
    return out


def tiles(mask_row_a, mask_row_b):
    u = mask_row_a if mask_row_b is None else (mask_row_a | mask_row_b)
    return (int(u.sum()) + 1) // 2


def run(w, p, sta, heads=None):
    og = P.geometry(w, heads=None if heads is None else len(heads))
    g = dbst.Geom.make(og.B, og.H, og.D, (og.T, og.Y, og.X), (og.tt, og.ty, og.tx))
    q, k, v = S.make_qkv(w, heads=heads)
    qd, kd, vd = (P.bits_to_torch(a) for a in (q, k, v))
    bits, cnt, idx = dbst.build_block_mask_raster(qd, kd, g, p, sta)
    pairs = dbst.pair_query_blocks(bits, g)
    pairs2 = dbst.pair_query_blocks(bits, g)
    dbst.get_error()
    mask = P.unpack_mask(bits.cpu().numpy().view(np.uint32), og.NB)
    return og, g, (q, k, v), (qd, kd, vd), (bits, cnt, idx), pairs, pairs2, mask


CASES = [("small", 0.9, 1, None), ("sweep", 0.7, -1, range(0, 16, 4)), ("wan", 0.9, -1, range(0, 40, 10)),
         ("hunyuan", 0.9, 1, range(0, 24, 12))]


@pytest.mark.parametrize("name,p,sta,heads", CASES)
def test_pairs_are_a_valid_cheaper_schedule(built, name, p, sta, heads):
    og, _, _, _, _, pairs, pairs2, mask = run(S.workload(name), p, sta, heads)
    assert torch.equal(pairs, pairs2), "pairing is not deterministic"
    qa, qb = decode(pairs)
    new_cost = fixed_cost = 0
    for b in range(og.B):
        for h in range(og.H):
            seen = np.zeros(og.NB, np.int64)
            for a_, b_ in zip(qa[b, h], qb[b, h]):
                assert a_ < og.NB and (b_ < og.NB or b_ == 0xFFFF)
                seen[a_] += 1
                if b_ != 0xFFFF:
                    seen[b_] += 1
                new_cost += tiles(mask[b, h, a_], None if b_ == 0xFFFF else mask[b, h, b_])
            assert (seen == 1).all(), "every block exactly once"
            assert (qb[b, h] == 0xFFFF).sum() == og.NB % 2
            for a_, b_ in fixed_pairs(og):
                fixed_cost += tiles(mask[b, h, a_], None if b_ is None else mask[b, h, b_])
    assert new_cost <= fixed_cost, (new_cost, fixed_cost)


@pytest.mark.parametrize("name,p,sta,heads", CASES[:2])
def test_attention_on_pairs_matches_oracle(built, name, p, sta, heads):
    w = S.workload(name)
    og, g, (q, k, v), (qd, kd, vd), (bits, cnt, idx), pairs, _, mask = run(w, p, sta, heads)
    o, lse = dbst.block_sparse_attn_raster(qd, kd, vd, g, cnt, idx, pairs=pairs)
    o_fixed, _ = dbst.block_sparse_attn_raster(qd, kd, vd, g, cnt, idx)
    dbst.get_error()
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    # the oracle on its own mask; outputs compared on the query blocks whose mask rows agree
    ref, _ = P.oracle_mask_per_head(qt, kt, og, p, sta)
    agree = (mask == ref).all(-1)
    assert agree.mean() >= 0.9
    sel = np.repeat(agree, 64, axis=-1)
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, ref, 64, 1.0 / math.sqrt(w.D))
    for got in (o, o_fixed):
        got_t = O.tile_reorder(got.float().cpu().numpy().astype(np.float64), og)
        max_abs, rel = P.attn_errors(got_t[sel], o_ref[sel])
        assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    lse_t = O.tile_reorder(lse.cpu().numpy()[..., None], og)[..., 0]
    assert np.max(np.abs(lse_t[sel] - lse_ref[sel])) <= P.LSE_MAX_ABS


def test_out_of_range_pair_entry_is_reported(built):
    w = S.workload("small")
    og, g, _, (qd, kd, vd), (bits, cnt, idx), pairs, _, _ = run(w, 0.9, 1)
    bad = pairs.clone()
    bad[0, 0, 0] = og.NB - 65536                # qa = NB (one past the last block), qb = 0xFFFF
    dbst.block_sparse_attn_raster(qd, kd, vd, g, cnt, idx, pairs=bad)
    with pytest.raises(dbst.DbstError) as e:
        dbst.get_error()
    assert e.value.status == dbst.DBST_EBOUNDS
