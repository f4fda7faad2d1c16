"""Bounded waits that run out: failure detection without a GPU fault.

Every wait between the roles of the attention kernels (forward and backward)
is bounded.  One that runs out records DBST_ETIMEOUT in the library's device
error word; the kernel then abandons its work, still waits (with the default
limit) for the copies and tensor-core products it issued, frees its tensor
memory and returns.  Here the limit is shortened with dbst_set_wait_limit so
that the first wait not satisfied at once runs out.  The call must report
DBST_ETIMEOUT through dbst_get_error, the CUDA context must stay usable, and
the very next call with the default limit, on the same stream, must agree
with the float64 oracle.
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

SHORT_LIMIT = 64   # SM cycles: shorter than any TMA copy or tensor-core product takes


@pytest.fixture(scope="module")
def built():
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    dbst.load()
    return True


def setup(name, p, sta):
    w = S.workload(name)
    og = P.geometry(w)
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    q, k, v = S.make_qkv(w)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    mask = O.build_block_mask(qt, kt, og, p, sta)
    words = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    cnt, idx = dbst.mask_from_bits(words, g)
    dbst.get_error()
    return w, og, g, (qt, kt, vt), mask, words, cnt, idx


def expect_timeout(fn):
    dbst.set_wait_limit(SHORT_LIMIT)
    try:
        fn()
        with pytest.raises(dbst.DbstError) as e:
            dbst.get_error()
        assert e.value.status == dbst.DBST_ETIMEOUT, e.value.status
    finally:
        dbst.set_wait_limit(0)
    dbst.get_error()   # the error word was cleared and nothing else is pending


# workloads with enough tiles per thread block that some wait cannot already be satisfied within the
# first test of the barrier (mbarrier.try_wait may itself suspend briefly until the phase completes)
@pytest.mark.parametrize("name,p,sta", [("small", 0.9, 1), ("small", 0.8, -1)])
def test_forward_wait_expiry_is_reported_and_the_next_call_is_exact(built, name, p, sta):
    w, og, g, (qt, kt, vt), mask, _, cnt, idx = setup(name, p, sta)
    tq, tk, tv = (P.bits_to_torch(a) for a in (qt, kt, vt))
    expect_timeout(lambda: dbst.block_sparse_attn(tq, tk, tv, g, cnt, idx))
    o, lse = dbst.block_sparse_attn(tq, tk, tv, g, cnt, idx)
    dbst.get_error()
    o_ref, lse_ref = O.masked_attention(qt, kt, vt, mask, 64, 1.0 / math.sqrt(w.D))
    max_abs, rel = P.attn_errors(o.float().cpu().numpy().astype(np.float64), o_ref)
    assert max_abs <= P.ATTN_MAX_ABS and rel <= P.ATTN_REL_L2, (max_abs, rel)
    lse = lse.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(lse - lse_ref)) <= P.LSE_MAX_ABS


def test_backward_wait_expiry_is_reported_and_the_next_call_is_exact(built):
    w, og, g, (qt, kt, vt), mask, words, cnt, idx = setup("small", 0.9, 1)
    tq, tk, tv = (P.bits_to_torch(a) for a in (qt, kt, vt))
    tdo = P.bits_to_torch(O.tile_reorder(S.make_grad(w), og))
    _, lse = dbst.block_sparse_attn(tq, tk, tv, g, cnt, idx)
    _, q_count, q_idx = dbst.transpose_block_mask(words, g)
    dbst.get_error()
    run = lambda: dbst.block_sparse_attn_backward(tq, tk, tv, lse, tdo, g, cnt, idx, q_count, q_idx)
    expect_timeout(run)
    dq, dk, dv = run()
    dbst.get_error()
    scale = 1.0 / math.sqrt(w.D)
    dot = S.f32_from_bf16_bits(P.torch_to_bits(tdo)).astype(np.float64)
    ref = O.masked_attention_backward(qt, kt, vt, mask, 64, scale, dot)
    for name, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        got = S.f32_from_bf16_bits(P.torch_to_bits(got)).astype(np.float64)
        assert np.linalg.norm(got - r) / np.linalg.norm(r) <= 1e-2, name
