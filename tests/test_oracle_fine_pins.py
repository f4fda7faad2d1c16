"""Pins of the fine-grained key-group oracle (AB-Attention page, section "Les
trois techniques", third technique): group pooling against closed forms, the
group size of a whole tile against the NABLA block mask, full selection against
dense attention, and the gathered attention against PyTorch with a token mask."""
import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(99)


def geom(H=2, D=16, grid=(2, 8, 16), tile=(1, 8, 8)):
    return O.Geometry(1, H, D, *grid, *tile)


def test_group_pooling_closed_form():
    """Keys constant within each group of 4 and zero queries but one channel: the map's logits
    are the group constants times the pooled query, so the map is their softmax."""
    g = geom(H=1, D=4)
    c = RNG.standard_normal(g.N // 4)
    k = np.zeros((1, 1, g.N, 4))
    k[0, 0, :, 0] = np.repeat(c, 4)
    q = np.zeros((1, 1, g.N, 4))
    q[0, 0, :, 0] = 1.0
    A = O.fine_score_map(q, k, g, 4, scale=1.0)
    e = np.exp(c - c.max())
    np.testing.assert_allclose(A[0, 0], np.broadcast_to(e / e.sum(), A[0, 0].shape), rtol=1e-13)
    np.testing.assert_allclose(A.sum(-1), 1.0, rtol=1e-14)


def test_whole_tile_groups_are_the_nabla_mask():
    g = geom()
    q, k = (RNG.standard_normal((1, 2, g.N, 16)) for _ in range(2))
    for p in (0.5, 0.9):
        np.testing.assert_array_equal(O.build_fine_mask(q, k, g, p, G=64), O.build_block_mask(q, k, g, p))


def test_full_selection_is_dense_attention():
    g = geom()
    q, k, v = (RNG.standard_normal((1, 2, g.N, 16)) for _ in range(3))
    mask = O.build_fine_mask(q, k, g, 1.0, G=4)
    assert mask.all()
    o, _ = O.fine_masked_attention(q, k, v, mask, 64, 4, 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a) for a in (q, k, v)), scale=0.25).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("G", [4, 8, 16])
def test_gathered_attention_equals_token_mask(G):
    g = geom()
    q, k, v = (RNG.standard_normal((1, 2, g.N, 16)) for _ in range(3))
    mask = RNG.random((1, 2, g.NB, g.N // G)) < 0.2
    mask[0, 0, 1] = False                                      # an empty row
    mask[0, 1, 0] = False
    mask[0, 1, 0, 5] = True                                    # a single group
    o, lse = O.fine_masked_attention(q, k, v, mask, 64, G, 0.3)
    tok = np.repeat(np.repeat(mask, 64, axis=2), G, axis=3)
    empty = ~tok.any(-1)
    safe = tok | empty[..., None]
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a) for a in (q, k, v)), attn_mask=torch.from_numpy(safe), scale=0.3).numpy()
    np.testing.assert_allclose(o[~empty], ref[~empty], rtol=1e-11, atol=1e-12)
    assert (o[empty] == 0).all() and np.isneginf(lse[empty]).all()


def test_group_size_must_divide_tile():
    g = geom()
    q = np.zeros((1, 2, g.N, 16))
    with pytest.raises(ValueError):
        O.fine_score_map(q, q, g, 3)


def test_kept_mass_meets_p():
    g = geom()
    q, k = (RNG.standard_normal((1, 2, g.N, 16)) * 2 for _ in range(2))
    mask, A = O.build_fine_mask(q, k, g, 0.8, G=4, return_scores=True)
    m = O.kept_mass(A, mask)
    assert (m >= 0.8 - 1e-12).all()
