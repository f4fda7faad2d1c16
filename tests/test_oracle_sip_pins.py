"""Pins of the SIP oracle (AB-Attention page, section "Les trois techniques",
SIP): inclusion probabilities against closed forms and their defining
properties, and unbiasedness of the weighted numerator and normaliser by
exact enumeration of every sample on tiny inputs."""
import itertools

import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(777)


def test_inclusion_probabilities_closed_forms():
    np.testing.assert_allclose(O.inclusion_probabilities_row([0.5, 0.3, 0.1, 0.1], 2), [1, 0.6, 0.2, 0.2],
                               rtol=1e-14)
    # one block above the cap: fixed at 1, the rest share the remaining budget of 1
    np.testing.assert_allclose(O.inclusion_probabilities_row([0.7, 0.1, 0.1, 0.1], 2), [1, 1 / 3, 1 / 3, 1 / 3],
                               rtol=1e-14)
    # a cascade: capping the first pushes the second over the cap as well
    np.testing.assert_allclose(O.inclusion_probabilities_row([0.6, 0.3, 0.05, 0.05], 3), [1, 1, 0.5, 0.5],
                               rtol=1e-14)
    # zero scores are never sampled; a budget covering every positive block keeps them all
    np.testing.assert_array_equal(O.inclusion_probabilities_row([0.0, 0.5, 0.5, 0.0], 3), [0, 1, 1, 0])
    np.testing.assert_array_equal(O.inclusion_probabilities_row([0.2, 0.3, 0.5], 3), [1, 1, 1])
    with pytest.raises(ValueError):
        O.inclusion_probabilities_row([0.5, -0.1], 1)
    with pytest.raises(ValueError):
        O.inclusion_probabilities_row([0.5, 0.5], 0)


@pytest.mark.parametrize("K", [1, 2.5, 4, 7])
def test_inclusion_probabilities_properties(K):
    A = RNG.dirichlet(np.full(12, 0.3), size=50)
    pi = O.inclusion_probabilities(A, K)
    assert ((pi >= 0) & (pi <= 1)).all()
    np.testing.assert_allclose(pi.sum(-1), np.minimum(K, (A > 0).sum(-1)), rtol=1e-12)
    for a, p in zip(A, pi):
        frac = (p > 0) & (p < 1)
        if frac.any():
            c = p[frac] / a[frac]
            np.testing.assert_allclose(c, c[0], rtol=1e-12)               # proportional to the score
            assert (a[p == 1] * c[0] >= 1 - 1e-12).all()                  # certain blocks are the top ones
            assert a[p == 1].min(initial=np.inf) >= a[frac].max()


def test_sampling_rule():
    pi = np.array([1.0, 0.5, 0.0, 0.25])
    np.testing.assert_array_equal(O.sip_sample(pi, [0.999, 0.49, 0.0, 0.25]), [True, True, False, False])


@pytest.mark.parametrize("K", [1.5, 2, 3])
def test_numerator_and_normaliser_are_unbiased(K):
    """For each query block, sum over all 2^NB samples of its row weighted by their probability:
    E[exp(lse)] equals the full softmax normaliser and E[exp(lse) * o] the full numerator
    (Horvitz-Thompson).  Rows are sampled independently, so each is enumerated on its own."""
    B, H, NB, blk, D, scale = 1, 1, 4, 2, 3, 0.6
    q, k, v = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(3))
    A = RNG.dirichlet(np.ones(NB), size=(B, H, NB))
    A[0, 0, 1, 2] = 0.0                                   # a zero score: never sampled
    A /= A.sum(-1, keepdims=True)
    pi = O.inclusion_probabilities(A, K)
    s = np.einsum("bhnd,bhmd->bhnm", q, k) * scale
    full_den = np.exp(s).sum(-1)
    full_num = np.einsum("bhnm,bhmd->bhnd", np.exp(s), v)
    for i in range(NB):
        rows = slice(i * blk, (i + 1) * blk)
        e_den = np.zeros(blk)
        e_num = np.zeros((blk, D))
        total = 0.0
        for pattern in itertools.product([False, True], repeat=NB):
            keep_row = np.array(pattern)
            prob = np.prod(np.where(keep_row, pi[0, 0, i], 1 - pi[0, 0, i]))
            total += prob
            if prob == 0.0:
                continue
            keep = np.zeros((B, H, NB, NB), bool)
            keep[0, 0, i] = keep_row
            o, lse = O.sip_attention(q, k, v, keep, pi, blk, scale)
            if keep_row.any():
                e_den += prob * np.exp(lse[0, 0, rows])
                e_num += prob * np.exp(lse[0, 0, rows])[:, None] * o[0, 0, rows]
        assert abs(total - 1.0) < 1e-12
        # a block with a zero score contributes nothing to the estimate: compare with the full
        # sums over the blocks that can be sampled
        cols = np.repeat(pi[0, 0, i] > 0, blk)
        den = np.exp(s[0, 0, rows][:, cols]).sum(-1)
        num = np.exp(s[0, 0, rows][:, cols]) @ v[0, 0][cols]
        np.testing.assert_allclose(e_den, den, rtol=1e-12)
        np.testing.assert_allclose(e_num, num, rtol=1e-11, atol=1e-12)
        if (pi[0, 0, i] > 0).all():
            np.testing.assert_allclose(e_den, full_den[0, 0, rows], rtol=1e-12)
            np.testing.assert_allclose(e_num, full_num[0, 0, rows], rtol=1e-11, atol=1e-12)


def test_every_block_certain_is_dense_attention():
    B, H, NB, blk, D = 1, 2, 3, 64, 16
    q, k, v = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(3))
    pi = np.ones((B, H, NB, NB))
    o, _ = O.sip_attention(q, k, v, np.ones_like(pi, bool), pi, blk, 0.25)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a) for a in (q, k, v)), scale=0.25).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_offset_equals_token_bias_in_torch():
    """Kept blocks with their log(1/pi) offsets = sdpa with an additive float mask."""
    B, H, NB, blk, D = 1, 1, 4, 16, 8
    q, k, v = (RNG.standard_normal((B, H, NB * blk, D)) for _ in range(3))
    pi = RNG.uniform(0.1, 1.0, size=(B, H, NB, NB))
    keep = RNG.random((B, H, NB, NB)) < 0.6
    keep[..., 0] = True
    o, _ = O.sip_attention(q, k, v, keep, pi, blk, 0.3)
    bias = np.where(keep, -np.log(pi), -np.inf)
    bias = np.repeat(np.repeat(bias, blk, axis=2), blk, axis=3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        *(torch.from_numpy(a) for a in (q, k, v)), attn_mask=torch.from_numpy(bias), scale=0.3).numpy()
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)
