"""Float64 oracle of the SQuad two-pass attention operator.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing in the library
imports it.

Source: "SQuad: Sub-Quadratic Attention Distillation for Efficient Video
Generation" (technical summary), section "Methodology: SQuad", item
"1. SQuad-Attention Operator" (the same operator is described in the French
summary of the page, section "1. Opérateur d'Attention SQuad").  Full softmax
attention is factorised into two passes over a sequence of n = m * w tokens:

* local pass Attn_L: each token attends, with an ordinary softmax, to the w
  tokens of its own window (windows are consecutive runs of w tokens);
* global pass Attn_G: each token attends to the m tokens that sit at the same
  position inside their windows, one per window;
* composition: the local pass's output is the value stream of the global
  pass; the global pass's output is the operator's output.

Readings where the page is silent:

S1  Queries and keys of both passes are the layer's own q and k; only the
    value stream of the global pass changes (to the local output).
S2  Windows are consecutive runs of w tokens of the sequence in the order the
    caller gives it; token t sits in window t // w at offset t % w.
S3  w divides n.  The page sets w = sqrt(n); any divisor is accepted here.
S4  Both passes use the same softmax scale (the attention's own, 1/sqrt(D) by
    default).
"""
from __future__ import annotations

import numpy as np

from .nabla import bf16_bits_to_f64


def _softmax(s: np.ndarray) -> np.ndarray:
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def squad_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, w: int, scale: float):
    """The SQuad operator on ``[B, H, n, D]`` inputs (bf16 bits or floats) with window w.

    Returns ``(o, o_local)``, float64 ``[B, H, n, D]``: the global pass output and the local
    pass output that fed its value stream.
    """
    dec = bf16_bits_to_f64 if q.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    B, H, n, D = q.shape
    if w < 1 or n % w:
        raise ValueError("the window must divide the sequence length")
    m = n // w
    # [B, H, window a, offset r, D]
    Q, K, V = (dec(x).reshape(B, H, m, w, D) for x in (q, k, v))
    # local pass: within window a, offset r attends to offsets r2 of the same window
    p_loc = _softmax(np.einsum("bhard,bhasd->bhars", Q, K) * scale)
    o_loc = np.einsum("bhars,bhasd->bhard", p_loc, V)
    # global pass: offset r of window a attends to offset r of every window c; values = local output
    p_glob = _softmax(np.einsum("bhard,bhcrd->bhrac", Q, K) * scale)
    o = np.einsum("bhrac,bhcrd->bhard", p_glob, o_loc)
    return o.reshape(B, H, n, D), o_loc.reshape(B, H, n, D)


def squad_flops(B: int, H: int, n: int, D: int, w: int) -> float:
    """Multiply-adds x 2 of the two passes: 4*D*n*w (local) + 4*D*n*(n/w) (global) per head."""
    return 4.0 * D * n * (w + n // w) * B * H
