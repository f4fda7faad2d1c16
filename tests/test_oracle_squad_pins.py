"""Pins of the SQuad oracle ("SQuad: Sub-Quadratic Attention Distillation for
Efficient Video Generation", section "Methodology: SQuad") against special
cases that reduce to ordinary attention and against PyTorch's attention with
explicit masks."""
import numpy as np
import pytest
import torch

import oracle as O

RNG = np.random.default_rng(4242)


def sdpa(q, k, v, scale, mask=None):
    t = [torch.from_numpy(np.ascontiguousarray(a)) for a in (q, k, v)]
    return torch.nn.functional.scaled_dot_product_attention(
        *t, attn_mask=None if mask is None else torch.from_numpy(mask), scale=scale).numpy()


def test_one_window_is_dense_attention():
    """w = n: the local pass is full attention and each global group holds one token."""
    q, k, v = (RNG.standard_normal((2, 2, 48, 8)) for _ in range(3))
    o, o_loc = O.squad_attention(q, k, v, 48, 0.3)
    ref = sdpa(q, k, v, 0.3)
    np.testing.assert_allclose(o_loc, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)


def test_unit_windows_make_the_global_pass_dense():
    """w = 1: the local pass returns v and the single global group is full attention."""
    q, k, v = (RNG.standard_normal((1, 3, 40, 8)) for _ in range(3))
    o, o_loc = O.squad_attention(q, k, v, 1, 0.25)
    np.testing.assert_array_equal(o_loc, v)
    np.testing.assert_allclose(o, sdpa(q, k, v, 0.25), rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("n,w", [(64, 8), (60, 12), (64, 16), (96, 4)])
def test_two_masked_attentions(n, w):
    """Local pass = attention under the same-window mask; global pass = attention under the
    same-offset mask with the local output as values."""
    q, k, v = (RNG.standard_normal((2, 2, n, 16)) * 2 for _ in range(3))
    t = np.arange(n)
    local = (t[:, None] // w) == (t[None, :] // w)
    glob = (t[:, None] % w) == (t[None, :] % w)
    o_loc_ref = sdpa(q, k, v, 0.2, local)
    o_ref = sdpa(q, k, o_loc_ref, 0.2, glob)
    o, o_loc = O.squad_attention(q, k, v, w, 0.2)
    np.testing.assert_allclose(o_loc, o_loc_ref, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(o, o_ref, rtol=1e-10, atol=1e-11)


def test_constant_values_pass_through():
    q, k = (RNG.standard_normal((1, 1, 64, 8)) * 3 for _ in range(2))
    c = RNG.standard_normal(8)
    v = np.broadcast_to(c, (1, 1, 64, 8))
    o, _ = O.squad_attention(q, k, v, 8, 0.5)
    np.testing.assert_allclose(o, np.broadcast_to(c, o.shape), rtol=1e-12, atol=1e-12)


def test_window_must_divide_length_and_flops():
    q = np.zeros((1, 1, 10, 4))
    with pytest.raises(ValueError):
        O.squad_attention(q, q, q, 3, 1.0)
    assert O.squad_flops(1, 1, 16384, 128, 128) == 4.0 * 128 * 16384 * 256
