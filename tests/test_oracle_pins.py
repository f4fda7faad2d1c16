"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each test checks one step of the NABLA path ("NABLA: Neighborhood Adaptive
Block-Level Attention", section "Méthodologie : NABLA") against brute force,
a closed form, an invariant stated by the method, or a library routine
(torch / scipy) computing the same textbook quantity.
"""
import itertools
import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle as O

RNG = np.random.default_rng(12345)


def geom(B=1, H=1, D=8, grid=(2, 8, 8), tile=(1, 8, 8)):
    return O.Geometry(B, H, D, *grid, *tile)


# --------------------------------------------------------------------------
# Token reorder ("Fractal Flattening")
# --------------------------------------------------------------------------

TILINGS = [((4, 8, 8), (1, 8, 8)), ((4, 8, 16), (2, 4, 8)), ((2, 16, 8), (2, 4, 8)),
           ((3, 8, 24), (1, 8, 8)), ((4, 4, 16), (4, 4, 4))]


@pytest.mark.parametrize("grid,tile", TILINGS)
def test_reorder_bruteforce(grid, tile):
    """Explicit coordinate walk: every token lands in its tile's contiguous run."""
    g = geom(B=1, H=2, D=3, grid=grid, tile=tile)
    T, Y, X = grid
    tt, ty, tx = tile
    nT, nY, nX = g.tile_grid
    x = RNG.integers(0, 2**16, size=(1, 2, g.N, 3), dtype=np.uint16)
    y = O.tile_reorder(x, g)
    for t in range(T):
        for yy in range(Y):
            for xx in range(X):
                tile_id = ((t // tt) * nY + (yy // ty)) * nX + (xx // tx)
                offset = ((t % tt) * ty + (yy % ty)) * tx + (xx % tx)
                src = (t * Y + yy) * X + xx
                np.testing.assert_array_equal(y[:, :, tile_id * g.blk + offset], x[:, :, src])


@pytest.mark.parametrize("grid,tile", TILINGS)
def test_reorder_roundtrip_and_tiles_are_boxes(grid, tile):
    g = geom(B=2, H=1, D=1, grid=grid, tile=tile)
    T, Y, X = grid
    coords = np.array([(t, yy, xx) for t in range(T) for yy in range(Y) for xx in range(X)])
    ids = np.arange(g.N, dtype=np.int64).reshape(1, 1, g.N, 1).repeat(2, axis=0)
    y = O.tile_reorder(ids, g)
    np.testing.assert_array_equal(O.tile_unreorder(y, g), ids)
    # every run of blk tiled tokens covers exactly one tt x ty x tx box
    for b in range(g.NB):
        c = coords[y[0, 0, b * g.blk:(b + 1) * g.blk, 0]]
        lo, hi = c.min(axis=0), c.max(axis=0)
        assert tuple(hi - lo + 1) == tuple(tile)
        assert all(lo[d] % tile[d] == 0 for d in range(3))
    # tiles are visited in raster order of tile coordinates (time order kept)
    first = coords[y[0, 0, ::g.blk, 0]] // np.array(tile)
    assert [tuple(r) for r in first] == sorted(tuple(r) for r in first)


# --------------------------------------------------------------------------
# Block mean-pool ("Sous-échantillonnage")
# --------------------------------------------------------------------------

def test_pool_blockwise_constant_is_exact():
    # bf16-representable values (8 significant bits): 64 copies sum exactly in fp64
    vals = RNG.integers(-255, 256, size=(2, 3, 5, 7)) * 2.0 ** RNG.integers(-12, 4, size=(2, 3, 5, 7))
    x = np.repeat(vals, 64, axis=2)
    np.testing.assert_array_equal(O.block_mean_pool(x, 64), vals)


def test_pool_linear_ramp_closed_form():
    n = np.arange(64 * 6, dtype=np.float64)
    x = (3.0 * n - 7.0).reshape(1, 1, -1, 1)
    expect = 3.0 * (64 * np.arange(6) + 31.5) - 7.0
    np.testing.assert_allclose(O.block_mean_pool(x, 64)[0, 0, :, 0], expect, rtol=0, atol=1e-12)


def test_pool_reads_bf16_bits_exactly():
    # 1.5 and -0.25 are exact in bf16; a block of alternating values has a known mean
    b = np.array([0x3FC0, 0xBE80], dtype=np.uint16)          # 1.5, -0.25
    x = np.tile(b, 32).reshape(1, 1, 64, 1)
    np.testing.assert_array_equal(O.block_mean_pool(O.bf16_bits_to_f64(x), 64), [[[[0.625]]]])


# --------------------------------------------------------------------------
# Reduced attention map ("Attention Réduite")
# --------------------------------------------------------------------------

def test_score_map_rows_sum_to_one_and_match_torch_softmax():
    qp = RNG.standard_normal((2, 3, 9, 16)) * 3
    kp = RNG.standard_normal((2, 3, 9, 16)) * 3
    A = O.pooled_score_map(qp, kp, 0.25)
    np.testing.assert_allclose(A.sum(-1), 1.0, rtol=0, atol=1e-14)
    ref = torch.softmax(torch.from_numpy(qp) @ torch.from_numpy(kp).transpose(-1, -2) * 0.25, dim=-1)
    np.testing.assert_allclose(A, ref.numpy(), rtol=1e-13, atol=1e-15)


def test_score_map_identical_keys_uniform_and_two_block_closed_form():
    qp = RNG.standard_normal((1, 1, 4, 8))
    kp = np.repeat(RNG.standard_normal((1, 1, 1, 8)), 6, axis=2)
    np.testing.assert_allclose(O.pooled_score_map(qp, kp, 1.0), 1.0 / 6, rtol=0, atol=1e-15)
    # two key blocks: A = logistic(s0 - s1)
    qp = np.array([[[[1.0, 0.0]]]])
    kp = np.array([[[[700.0, 0.0], [697.0, 1.0]]]])          # logits 700 and 697: no overflow allowed
    A = O.pooled_score_map(qp, kp, 1.0)[0, 0, 0]
    np.testing.assert_allclose(A, [1 / (1 + math.exp(-3.0)), 1 / (1 + math.exp(3.0))], rtol=1e-14)


# --------------------------------------------------------------------------
# CDF threshold ("Seuil CDF")
# --------------------------------------------------------------------------

def _rows(n, nb, conc=0.3):
    return RNG.dirichlet(np.full(nb, conc), size=n)


@pytest.mark.parametrize("p", [0.05, 0.5, 0.8, 0.9, 0.95, 0.999])
def test_cdf_mass_reaches_p_and_set_is_minimal(p):
    for a in _rows(200, 37):
        keep = O.cdf_select_row(a, p)
        mass = a[keep].sum()
        assert mass >= p
        assert mass - a[keep].min() < p                      # dropping the smallest kept block falls below p
        assert a[keep].min() >= a[~keep].max(initial=0.0)     # kept blocks are the largest ones


def test_cdf_p_one_keeps_all_and_tiny_p_keeps_argmax():
    for a in _rows(50, 20):
        assert O.cdf_select_row(a, 1.0).all()
        keep = O.cdf_select_row(a, 1e-12)
        assert keep.sum() == 1 and keep[np.argmax(a)]
    # exact tie at the top: the lower index wins
    a = np.array([0.1, 0.35, 0.35, 0.2])
    assert list(np.nonzero(O.cdf_select_row(a, 0.3))[0]) == [1]
    assert list(np.nonzero(O.cdf_select_row(a, 0.36))[0]) == [1, 2]


@pytest.mark.parametrize("nb", [3, 5, 8])
def test_cdf_bruteforce_over_all_subsets(nb):
    """Greedy CDF prefix == the smallest subset reaching p, and the heaviest of that size."""
    for a in _rows(60, nb, conc=0.7):
        for p in (0.3, 0.6, 0.9):
            keep = O.cdf_select_row(a, p)
            best_k, best_mass, best_set = None, -1.0, None
            for k in range(1, nb + 1):
                for sub in itertools.combinations(range(nb), k):
                    m = a[list(sub)].sum()
                    if m >= p and m > best_mass:
                        best_mass, best_set = m, set(sub)
                if best_set is not None:
                    best_k = k
                    break
            assert keep.sum() == best_k
            assert set(np.nonzero(keep)[0]) == best_set


def test_cdf_matches_page_ascending_form():
    """The page's wording: ascending CDF, keep blocks whose cumulative mass exceeds 1 - p."""
    for p in (0.5, 0.8, 0.9, 0.95):
        for a in _rows(300, 48):
            desc = np.sort(a)[::-1]
            if np.min(np.abs(np.cumsum(desc) - p)) < 1e-9:
                continue                                      # too close to call in fp64
            order = np.argsort(a, kind="stable")              # ascending
            c = np.cumsum(a[order])
            page_keep = np.zeros_like(a, dtype=bool)
            page_keep[order[c > 1.0 - p]] = True
            np.testing.assert_array_equal(O.cdf_select_row(a, p), page_keep)


def test_build_mask_rejects_bad_p():
    g = geom()
    x = np.zeros((1, 1, g.N, g.D))
    for p in (0.0, -0.1, 1.5):
        with pytest.raises(ValueError):
            O.build_block_mask(x, x, g, p)


# --------------------------------------------------------------------------
# Sliding-tile neighbourhood and the union ("Intégration Hybride avec STA")
# --------------------------------------------------------------------------

@pytest.mark.parametrize("grid,tile", [((8, 16, 16), (1, 8, 8)), ((8, 16, 32), (2, 4, 8))])
@pytest.mark.parametrize("r", [0, 1, 2])
def test_sta_neighbour_sets_bruteforce(grid, tile, r):
    g = geom(grid=grid, tile=tile)
    nT, nY, nX = g.tile_grid
    M = O.sta_mask(g, r)
    cells = list(itertools.product(range(nT), range(nY), range(nX)))
    for i, ci in enumerate(cells):
        expect = {j for j, cj in enumerate(cells) if all(abs(a - b) <= r for a, b in zip(ci, cj))}
        assert set(np.nonzero(M[i])[0]) == expect
    assert (M == M.T).all() and M.diagonal().all()


def test_sta_large_radius_is_all_ones_and_negative_is_empty():
    g = geom(grid=(4, 16, 16), tile=(1, 8, 8))
    assert O.sta_mask(g, 10).all()
    assert not O.sta_mask(g, -1).any()


def test_build_mask_union_and_p1():
    g = geom(B=1, H=2, D=16, grid=(4, 16, 16), tile=(1, 8, 8))
    q = RNG.standard_normal((1, 2, g.N, 16)) * 2
    k = RNG.standard_normal((1, 2, g.N, 16)) * 2
    assert O.build_block_mask(q, k, g, 1.0).all()
    m_plain = O.build_block_mask(q, k, g, 0.5)
    m_sta = O.build_block_mask(q, k, g, 0.5, sta_radius=1)
    np.testing.assert_array_equal(m_sta, m_plain | O.sta_mask(g, 1)[None, None])


def test_mask_to_lists_ascending_and_counts():
    m = RNG.random((2, 2, 9, 9)) < 0.4
    m[0, 0, 3] = False
    cnt, idx = O.mask_to_lists(m)
    for b, h, i in itertools.product(range(2), range(2), range(9)):
        js = list(np.nonzero(m[b, h, i])[0])
        assert cnt[b, h, i] == len(js)
        assert list(idx[b, h, i, :len(js)]) == js


# --------------------------------------------------------------------------
# Attention over the kept blocks ("Expansion")
# --------------------------------------------------------------------------

def _sdpa(q, k, v, keep_tokens, scale):
    qt, kt, vt = (torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v))
    return torch.nn.functional.scaled_dot_product_attention(
        qt, kt, vt, attn_mask=torch.from_numpy(keep_tokens), scale=scale).numpy()


def test_masked_attention_matches_torch_sdpa_with_expanded_mask():
    B, H, NB, blk, D = 1, 2, 5, 64, 16
    q = RNG.standard_normal((B, H, NB * blk, D))
    k = RNG.standard_normal((B, H, NB * blk, D))
    v = RNG.standard_normal((B, H, NB * blk, D))
    mask = RNG.random((B, H, NB, NB)) < 0.5
    mask[0, 0, 2] = False                                     # one fully masked query block
    mask[0, 1, 4] = False
    mask[0, 1, 4, 1] = True                                   # a single kept block
    o, lse = O.masked_attention(q, k, v, mask, blk, 0.3)
    tok = np.repeat(np.repeat(mask, blk, axis=2), blk, axis=3)
    ref = _sdpa(q, k, v, tok, 0.3)
    empty = ~mask.any(-1)
    rows = np.repeat(empty, blk, axis=2)
    np.testing.assert_allclose(o[~rows], ref[~rows], rtol=1e-11, atol=1e-12)
    assert (o[rows] == 0).all() and np.isneginf(lse[rows]).all()
    # log-sum-exp of the kept logits, via scipy
    s = np.einsum("bhnd,bhmd->bhnm", q, k) * 0.3
    s = np.where(tok, s, -np.inf)
    with np.errstate(divide="ignore"):
        ref_lse = logsumexp(s, axis=-1)
    np.testing.assert_allclose(lse[~rows], ref_lse[~rows], rtol=1e-12)


def test_dense_equals_all_ones_mask_and_sdpa():
    B, H, N, D = 1, 1, 192, 32
    q, k, v = (RNG.standard_normal((B, H, N, D)) for _ in range(3))
    o_d, lse_d = O.dense_attention(q, k, v, 0.2)
    o_m, lse_m = O.masked_attention(q, k, v, np.ones((B, H, 3, 3), bool), 64, 0.2)
    np.testing.assert_allclose(o_d, o_m, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse_d, lse_m, rtol=1e-13)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a) for a in (q, k, v)), scale=0.2).numpy()
    np.testing.assert_allclose(o_d, ref, rtol=1e-11, atol=1e-12)


def test_constant_v_is_reproduced_whatever_the_mask():
    B, H, NB, blk, D = 1, 1, 4, 64, 8
    q = RNG.standard_normal((B, H, NB * blk, D)) * 4
    k = RNG.standard_normal((B, H, NB * blk, D)) * 4
    const = RNG.standard_normal(D)
    v = np.broadcast_to(const, (B, H, NB * blk, D))
    mask = RNG.random((B, H, NB, NB)) < 0.6
    mask[..., 0] = True
    o, _ = O.masked_attention(q, k, v, mask, blk, 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(const, o.shape), rtol=1e-12, atol=1e-12)


def test_single_kept_block_is_dense_attention_over_that_block():
    B, H, NB, blk, D = 1, 1, 6, 64, 16
    q, k, v = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(3))
    pick = RNG.integers(0, NB, size=NB)
    mask = np.zeros((B, H, NB, NB), bool)
    mask[0, 0, np.arange(NB), pick] = True
    o, _ = O.masked_attention(q, k, v, mask, blk, 0.25)
    for i in range(NB):
        sl = slice(pick[i] * blk, (pick[i] + 1) * blk)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q[:, :, i * blk:(i + 1) * blk]), torch.from_numpy(k[:, :, sl]),
            torch.from_numpy(v[:, :, sl]), scale=0.25).numpy()
        np.testing.assert_allclose(o[:, :, i * blk:(i + 1) * blk], ref, rtol=1e-11, atol=1e-12)


def test_row_subset_equals_full_computation():
    B, H, NB, blk, D = 1, 2, 4, 64, 8
    q, k, v = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(3))
    mask = RNG.random((B, H, NB, NB)) < 0.5
    o, lse = O.masked_attention(q, k, v, mask, blk, 0.4)
    rows = [(0, 1, 3), (0, 0, 0)]
    o_s, lse_s = O.masked_attention(q, k, v, mask, blk, 0.4, rows=rows)
    for r, (b, h, i) in enumerate(rows):
        np.testing.assert_array_equal(o_s[r], o[b, h, i * blk:(i + 1) * blk])
        np.testing.assert_array_equal(lse_s[r], lse[b, h, i * blk:(i + 1) * blk])


def test_end_to_end_p1_is_dense_attention():
    g = geom(B=1, H=2, D=16, grid=(2, 8, 16), tile=(1, 8, 8))
    q, k, v = (RNG.standard_normal((1, 2, g.N, 16)) for _ in range(3))
    qt, kt, vt = (O.tile_reorder(a, g) for a in (q, k, v))
    mask = O.build_block_mask(qt, kt, g, 1.0)
    o, _ = O.masked_attention(qt, kt, vt, mask, g.blk, 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a) for a in (q, k, v)), scale=0.25).numpy()
    np.testing.assert_allclose(O.tile_unreorder(o, g), ref, rtol=1e-11, atol=1e-12)


def test_cdf_select_batched_rows():
    """The batched selection keeps, per row, what the row selection keeps; p = 1 keeps every
    block; a one-hot row keeps exactly its hot block at any p."""
    A = RNG.random((2, 3, 5, 5))
    A /= A.sum(-1, keepdims=True)
    for p in (0.3, 0.9):
        got = O.cdf_select(A, p)
        assert got.shape == A.shape
        for idx in itertools.product(range(2), range(3), range(5)):
            np.testing.assert_array_equal(got[idx], O.cdf_select_row(A[idx], p))
    assert O.cdf_select(A, 1.0).all()
    hot = np.zeros((4, 4))
    hot[np.arange(4), [2, 0, 3, 1]] = 1.0
    for p in (0.01, 0.5, 0.999):
        sel = O.cdf_select(hot, p)
        np.testing.assert_array_equal(sel, hot > 0)


def test_kept_pair_flops_full_lists_equal_dense_flops():
    """Every list full: 4 * D * N^2 * B * H, the dense attention FLOP count."""
    B, H, D, NB = 2, 3, 128, 7
    kv_count = np.full((B, H, NB), NB, dtype=np.int32)
    N = NB * 64
    assert O.kept_pair_flops(kv_count, D) == 4.0 * D * N * N * B * H
    kv_count[0, 0, 0] = 0
    assert O.kept_pair_flops(kv_count, D) == 4.0 * D * N * N * B * H - 4.0 * D * NB * 64 * 64


# --------------------------------------------------------------------------
# Backward of the block-sparse attention (gradient of the forward definition)
# --------------------------------------------------------------------------

def _loss(q, k, v, mask, blk, scale, do):
    o, _ = O.masked_attention(q, k, v, mask, blk, scale)
    return float(np.sum(o * do))


def test_backward_matches_central_finite_differences():
    """d/dx of sum(o * do) by central differences, every element of q, k and v."""
    B, H, NB, blk, D, scale = 1, 2, 3, 2, 3, 0.7
    q, k, v, do = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(4))
    mask = np.array([[[[1, 0, 1], [0, 0, 0], [1, 1, 1]],
                      [[0, 1, 0], [1, 1, 0], [0, 0, 1]]]], dtype=bool)
    grads = O.masked_attention_backward(q, k, v, mask, blk, scale, do)
    h = 1e-6
    for which, g in enumerate(grads):
        args = [q, k, v]
        for idx in np.ndindex(q.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            fd = (_loss(*plus, mask, blk, scale, do) - _loss(*minus, mask, blk, scale, do)) / (2 * h)
            assert abs(fd - g[idx]) < 1e-7 * (1 + abs(fd)), (which, idx, fd, g[idx])


def _torch_grads(q, k, v, tok, scale, do):
    t = [torch.from_numpy(a.copy()).requires_grad_(True) for a in (q, k, v)]
    o = torch.nn.functional.scaled_dot_product_attention(
        *t, attn_mask=None if tok is None else torch.from_numpy(tok), scale=scale)
    o.backward(torch.from_numpy(do))
    return [x.grad.numpy() for x in t]


def test_backward_full_mask_equals_dense_autograd():
    B, H, NB, blk, D = 1, 2, 3, 64, 16
    q, k, v, do = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(4))
    got = O.masked_attention_backward(q, k, v, np.ones((B, H, NB, NB), bool), blk, 0.25, do)
    for g, r in zip(got, _torch_grads(q, k, v, None, 0.25, do)):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-12)


def test_backward_sparse_mask_equals_autograd_with_expanded_mask():
    B, H, NB, blk, D = 1, 2, 4, 64, 8
    q, k, v, do = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(4))
    mask = RNG.random((B, H, NB, NB)) < 0.4
    mask[..., np.arange(NB), np.arange(NB)] = True            # no empty row (sdpa would give NaN)
    tok = np.repeat(np.repeat(mask, blk, axis=2), blk, axis=3)
    got = O.masked_attention_backward(q, k, v, mask, blk, 0.3, do)
    for g, r in zip(got, _torch_grads(q, k, v, tok, 0.3, do)):
        np.testing.assert_allclose(g, r, rtol=1e-10, atol=1e-12)


def test_backward_empty_row_has_no_gradient_and_gives_none():
    """A query block with no kept key block: zero dq, and its do moves no dk / dv."""
    B, H, NB, blk, D = 1, 1, 3, 4, 5
    q, k, v, do = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(4))
    mask = np.ones((B, H, NB, NB), bool)
    mask[0, 0, 1] = False
    dq, dk, dv = O.masked_attention_backward(q, k, v, mask, blk, 0.5, do)
    assert (dq[0, 0, blk:2 * blk] == 0).all()
    do2 = do.copy()
    do2[0, 0, blk:2 * blk] = RNG.standard_normal((blk, D)) * 10
    dq2, dk2, dv2 = O.masked_attention_backward(q, k, v, mask, blk, 0.5, do2)
    np.testing.assert_array_equal(dk, dk2)
    np.testing.assert_array_equal(dv, dv2)
    np.testing.assert_array_equal(dq, dq2)


def test_backward_single_kept_key_closed_form():
    """One key per block and one kept block per row: softmax is 1, so dq = 0, dk = 0 and
    the kept key's dv is the sum of do over the rows that keep it."""
    B, H, NB, blk, D = 1, 1, 5, 1, 4
    q, k, v, do = (RNG.standard_normal((B, H, NB, D)) for _ in range(4))
    pick = np.array([3, 0, 3, 4, 3])
    mask = np.zeros((B, H, NB, NB), bool)
    mask[0, 0, np.arange(NB), pick] = True
    dq, dk, dv = O.masked_attention_backward(q, k, v, mask, blk, 0.9, do)
    assert np.abs(dq).max() < 1e-15 and np.abs(dk).max() < 1e-15
    ref = np.zeros((NB, D))
    np.add.at(ref, pick, do[0, 0])
    np.testing.assert_allclose(dv[0, 0], ref, rtol=1e-15, atol=1e-15)


def test_backward_is_linear_in_do_and_reads_bf16_bits():
    B, H, NB, blk, D = 1, 1, 3, 8, 4
    q, k, v = (torch.randn(B, H, NB * blk, D, dtype=torch.bfloat16,
                           generator=torch.Generator().manual_seed(s)) for s in (1, 2, 3))
    bits = [a.view(torch.int16).numpy().view(np.uint16) for a in (q, k, v)]
    f = [a.double().numpy() for a in (q, k, v)]
    mask = RNG.random((B, H, NB, NB)) < 0.6
    mask[..., 0] = True
    d1, d2 = RNG.standard_normal((2, B, H, NB * blk, D))
    g1 = O.masked_attention_backward(*bits, mask, blk, 0.5, d1)
    g2 = O.masked_attention_backward(*bits, mask, blk, 0.5, d2)
    g12 = O.masked_attention_backward(*bits, mask, blk, 0.5, 2 * d1 - 3 * d2)
    gf = O.masked_attention_backward(*f, mask, blk, 0.5, d1)
    for a, b, c, e in zip(g1, g2, g12, gf):
        np.testing.assert_allclose(c, 2 * a - 3 * b, rtol=1e-12, atol=1e-12)
        np.testing.assert_array_equal(a, e)


def test_backward_blocks_equal_full_backward():
    """The sampled-block form returns the full function's values for the chosen blocks (including
    a query block with an empty list and a key block nobody keeps)."""
    B, H, NB, blk, D = 2, 2, 5, 8, 4
    q, k, v, do = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(4))
    mask = RNG.random((B, H, NB, NB)) < 0.5
    mask[0, 1, 3] = False
    mask[1, 0, :, 2] = False
    dq, dk, dv = O.masked_attention_backward(q, k, v, mask, blk, 0.4, do)
    qs = [(0, 1, 3), (1, 1, 0), (0, 0, 4)]
    ks = [(1, 0, 2), (0, 1, 1), (1, 1, 4), (0, 1, 0)]
    gq, gkv = O.masked_attention_backward_blocks(q, k, v, mask, blk, 0.4, do, qs, ks)
    for b, h, i in qs:
        np.testing.assert_allclose(gq[(b, h, i)], dq[b, h, i * blk:(i + 1) * blk], rtol=1e-12, atol=1e-14)
    for b, h, j in ks:
        np.testing.assert_allclose(gkv[(b, h, j)][0], dk[b, h, j * blk:(j + 1) * blk], rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(gkv[(b, h, j)][1], dv[b, h, j * blk:(j + 1) * blk], rtol=1e-12, atol=1e-14)
    assert not gq[(0, 1, 3)].any() and not gkv[(1, 0, 2)][0].any() and not gkv[(1, 0, 2)][1].any()
