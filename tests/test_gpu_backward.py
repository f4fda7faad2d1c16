"""GPU parity of the block-sparse attention backward against the float64 oracle.

The backward is the exact gradient of the forward definition (dq, dk, dv over
the kept blocks); the oracle is ``oracle.masked_attention_backward``.  Both
sides use the same mask: the oracle's mask, packed and expanded to lists on
the GPU (``mask_from_bits``), so the comparison isolates the backward.

Bounds: P and dS are rounded to bf16 before the tensor-core products and the
outputs are bf16; an emulation of exactly that rounding on the tiny and small
workloads gives relative L2 errors up to 4.2e-3 and max-abs errors up to
7.2e-3 of max|ref|.  The tests allow 1e-2 and 2e-2.
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

GRAD_REL_L2 = 1e-2
GRAD_MAX_REL = 2e-2


@pytest.fixture(scope="module")
def built():
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    dbst.load()
    return True


def gpu_geom(w):
    return dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)


def f64(bits):
    return S.f32_from_bf16_bits(bits).astype(np.float64)


def check_grad(name, got_bits, ref):
    got = f64(got_bits)
    scale = np.abs(ref).max()
    if scale == 0:
        np.testing.assert_array_equal(got, 0.0, err_msg=name)
        return
    err = np.abs(got - ref)
    rel = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    assert err.max() <= GRAD_MAX_REL * scale, (name, err.max(), scale)
    assert rel <= GRAD_REL_L2, (name, rel)


def run_backward(w, q, k, v, do, mask, raster=False, scale=0.0):
    """GPU forward (for lse) and backward on the oracle's mask.  q, k, v, do: raster bf16 bits."""
    g = gpu_geom(w)
    og = P.geometry(w)
    bits = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    kv_count, kv_idx = dbst.mask_from_bits(bits, g)
    _, q_count, q_idx = dbst.transpose_block_mask(bits, g)
    if raster:
        tq, tk, tv, tdo = (P.bits_to_torch(a) for a in (q, k, v, do))
        _, lse = dbst.block_sparse_attn_raster(tq, tk, tv, g, kv_count, kv_idx, scale=scale)
    else:
        tq, tk, tv, tdo = (P.bits_to_torch(O.tile_reorder(a, og)) for a in (q, k, v, do))
        _, lse = dbst.block_sparse_attn(tq, tk, tv, g, kv_count, kv_idx, scale=scale)
    grads = dbst.block_sparse_attn_backward(tq, tk, tv, lse, tdo, g, kv_count, kv_idx, q_count, q_idx,
                                            scale=scale, raster=raster)
    dbst.get_error()
    return grads


def oracle_grads(w, q, k, v, do, mask, scale):
    og = P.geometry(w)
    qt, kt, vt = (O.tile_reorder(a, og) for a in (q, k, v))
    dot = f64(O.tile_reorder(do, og))
    return O.masked_attention_backward(qt, kt, vt, mask, 64, scale, dot)


def inputs(w):
    q, k, v = S.make_qkv(w)
    return q, k, v, S.make_grad(w)


# ---------------------------------------------------------------- transpose
@pytest.mark.parametrize("nb_grid", [((4, 8, 8), (1, 8, 8)), ((3, 16, 40), (1, 8, 8)), ((8, 16, 16), (2, 4, 8))])
def test_transpose_block_mask_is_exact(built, nb_grid):
    grid, tile = nb_grid
    w = S.Workload("t", 0, B=2, H=2, D=64, grid=grid, tile=tile, alpha=0.7, beta=0.3, f_rms=1.0, kmax=1,
                   p_list=(0.9,), sta_radius=-1)
    g = gpu_geom(w)
    rng = np.random.default_rng(7)
    mask = rng.random((2, 2, g.NB, g.NB)) < 0.3
    mask[0, 0, 1] = False            # a query block keeping nothing
    mask[0, 1, :, 2] = False         # a key block kept by nobody
    mask[1, 0] = True                # a full head
    bits = torch.from_numpy(P.pack_mask(mask).view(np.int32)).cuda()
    bits_t, q_count, q_idx = dbst.transpose_block_mask(bits, g)
    dbst.get_error()
    mt = np.swapaxes(mask, -1, -2)
    np.testing.assert_array_equal(bits_t.cpu().numpy().view(np.uint32), P.pack_mask(mt))
    cnt_ref, idx_ref = O.mask_to_lists(mt)
    cnt = q_count.cpu().numpy()
    idx = q_idx.cpu().numpy()
    np.testing.assert_array_equal(cnt, cnt_ref)
    for bhj in np.ndindex(cnt.shape):
        np.testing.assert_array_equal(idx[bhj][:cnt[bhj]], idx_ref[bhj][:cnt[bhj]])


# ---------------------------------------------------------------- parity
@pytest.mark.parametrize("name,p,D", [("tiny", 0.9, 64), ("tiny", 1.0, 128), ("small", 0.9, 64),
                                      ("small", 0.5, 128), ("small", 0.95, 64)])
def test_backward_matches_oracle(built, name, p, D):
    w = dataclasses.replace(S.workload(name), D=D)
    if name == "small":
        w = dataclasses.replace(w, H=4)
    q, k, v, do = inputs(w)
    og = P.geometry(w)
    mask = O.build_block_mask(O.tile_reorder(q, og), O.tile_reorder(k, og), og, p)
    dq, dk, dv = run_backward(w, q, k, v, do, mask)
    ref = oracle_grads(w, q, k, v, do, mask, 1.0 / np.sqrt(D))
    for nm, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        check_grad(f"{name} p={p} D={D} {nm}", P.torch_to_bits(got), r)


@pytest.mark.parametrize("D", [64, 128])
def test_backward_edge_masks(built, D):
    """Empty query rows, key blocks nobody keeps, single blocks, a full row, an odd block count
    (a CTA whose second block does not exist) and an explicit scale."""
    w = S.Workload("edge", 0, B=1, H=3, D=D, grid=(3, 16, 16), tile=(1, 8, 8), alpha=0.7, beta=0.3, f_rms=2.0,
                   kmax=2, p_list=(0.9,), sta_radius=-1)
    og = P.geometry(w)
    q, k, v, do = inputs(w)
    rng = np.random.default_rng(11)
    mask = rng.random((1, 3, og.NB, og.NB)) < 0.4
    mask[0, 0, 0] = False                          # query block 0 keeps nothing
    mask[0, 0, 5] = False
    mask[0, 0, 5, 7] = True                        # a single kept block
    mask[0, 0, :, 3] = False                       # key block 3 kept by nobody
    mask[0, 1, 2] = True                           # a full row
    mask[0, 2] = False                             # a head with nothing kept at all
    dq, dk, dv = run_backward(w, q, k, v, do, mask, scale=0.2)
    ref = oracle_grads(w, q, k, v, do, mask, 0.2)
    for nm, got, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        check_grad(f"edge D={D} {nm}", P.torch_to_bits(got), r)
    gq, gk, gv = (P.torch_to_bits(t) for t in (dq, dk, dv))
    assert not gq[0, 0, :64].any() and not gq[0, 2].any()          # tiled rows of block 0; empty head
    assert not gk[0, 0, 3 * 64:4 * 64].any() and not gv[0, 0, 3 * 64:4 * 64].any()
    assert not gk[0, 2].any() and not gv[0, 2].any()


def test_backward_raster_equals_tiled_bit_for_bit(built):
    w = dataclasses.replace(S.workload("small"), H=2, D=128)
    og = P.geometry(w)
    q, k, v, do = inputs(w)
    mask = O.build_block_mask(O.tile_reorder(q, og), O.tile_reorder(k, og), og, 0.9)
    tiled = run_backward(w, q, k, v, do, mask)
    raster = run_backward(w, q, k, v, do, mask, raster=True)
    for a, b in zip(tiled, raster):
        np.testing.assert_array_equal(O.tile_unreorder(P.torch_to_bits(a), og), P.torch_to_bits(b))


def test_backward_is_deterministic(built):
    w = dataclasses.replace(S.workload("small"), H=2)
    og = P.geometry(w)
    q, k, v, do = inputs(w)
    mask = O.build_block_mask(O.tile_reorder(q, og), O.tile_reorder(k, og), og, 0.9)
    first = [P.torch_to_bits(t) for t in run_backward(w, q, k, v, do, mask)]
    for _ in range(5):
        again = [P.torch_to_bits(t) for t in run_backward(w, q, k, v, do, mask)]
        for a, b in zip(first, again):
            np.testing.assert_array_equal(a, b)


def test_backward_on_gpu_built_mask(built):
    """The path as a training step runs it: GPU mask, its transpose, forward, backward."""
    w = dataclasses.replace(S.workload("small"), H=2, D=128)
    og = P.geometry(w)
    g = gpu_geom(w)
    q, k, v, do = inputs(w)
    tq, tk, tv, tdo = (P.bits_to_torch(a) for a in (q, k, v, do))
    bits, kv_count, kv_idx = dbst.build_block_mask_raster(tq, tk, g, 0.9)
    _, q_count, q_idx = dbst.transpose_block_mask(bits, g)
    _, lse = dbst.block_sparse_attn_raster(tq, tk, tv, g, kv_count, kv_idx)
    grads = dbst.block_sparse_attn_backward(tq, tk, tv, lse, tdo, g, kv_count, kv_idx, q_count, q_idx, raster=True)
    dbst.get_error()
    mask = P.unpack_mask(bits.cpu().numpy().view(np.uint32), og.NB)
    ref = oracle_grads(w, q, k, v, do, mask, 1.0 / np.sqrt(128))
    for nm, got, r in zip(("dq", "dk", "dv"), grads, ref):
        check_grad(nm, O.tile_reorder(P.torch_to_bits(got), og), r)
