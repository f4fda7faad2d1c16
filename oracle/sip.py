"""Float64 oracle of AB-Attention's sampled key-block selection (SIP).

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing in the library
imports it.

Source: "AB-Attention accélère la génération vidéo jusqu'à 2,23× en sautant 92%
de l'attention" (news.hamidun.com), section "Les trois techniques", second
technique, SIP (Sampling with Inclusion-Probability Weighting): instead of a
hard top-k, each key block enters the sample with probability proportional to
its score, the highest-scoring blocks always enter, and every kept block is
weighted by the inverse of its inclusion probability (Horvitz-Thompson), which
makes the softmax numerator and normaliser unbiased; the computation stays
ordinary softmax attention with a logit offset.

Readings where the page is silent:

A1  Scores are the rows of the NABLA pooled map (the softmax of the pooled
    logits, ``oracle.nabla.pooled_score_map``); AB-Attention's own scorer
    (IBCS) is out of scope.
A2  Inclusion probabilities: pi_j = min(1, c * a_j) with c chosen so that
    sum_j pi_j = K, the budget (expected number of kept blocks per row).  c is
    found by the usual fixed point: blocks with c * a_j >= 1 are fixed at 1 and
    c is recomputed over the rest with the remaining budget.  If K is at least
    the number of blocks with a_j > 0, all of those get pi_j = 1; blocks with
    a_j = 0 get pi_j = 0.
A3  Sampling is independent per block (Poisson sampling): block j is kept iff
    u_j < pi_j for a caller-supplied uniform u_j in [0, 1).  pi_j = 1 always
    keeps, pi_j = 0 never does.
A4  The offset of a kept block is log(1 / pi_j) (natural log), added to the
    scaled logits of all its keys.
"""
from __future__ import annotations

import numpy as np

from .nabla import bf16_bits_to_f64


def inclusion_probabilities_row(a: np.ndarray, K: float) -> np.ndarray:
    """pi for one row of non-negative scores and budget K (reading A2)."""
    a = np.asarray(a, dtype=np.float64)
    if (a < 0).any() or not np.isfinite(a).all():
        raise ValueError("scores must be finite and non-negative")
    if not K > 0:
        raise ValueError("the budget must be positive")
    pi = np.zeros_like(a)
    positive = a > 0
    if K >= positive.sum():
        pi[positive] = 1.0
        return pi
    certain = np.zeros(a.shape, dtype=bool)
    while True:
        rest = positive & ~certain
        c = (K - certain.sum()) / a[rest].sum()
        new = rest & (c * a >= 1.0)
        if not new.any():
            pi[rest] = c * a[rest]
            break
        certain |= new
    pi[certain] = 1.0
    return pi


def inclusion_probabilities(A: np.ndarray, K: float) -> np.ndarray:
    """pi for every row of ``A [..., NB]``."""
    flat = A.reshape(-1, A.shape[-1])
    out = np.stack([inclusion_probabilities_row(r, K) for r in flat])
    return out.reshape(A.shape)


def sip_sample(pi: np.ndarray, u: np.ndarray) -> np.ndarray:
    """Kept blocks: u < pi (reading A3)."""
    return np.asarray(u) < np.asarray(pi)


def sip_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, keep: np.ndarray, pi: np.ndarray, blk: int,
                  scale: float):
    """Attention of every query block over its kept key blocks, each kept block's logits offset
    by log(1/pi) (reading A4).  q, k, v ``[B, H, N, D]`` tile-ordered (bf16 bits or floats);
    keep, pi ``[B, H, NB, NB]``.  Returns (o, lse) float64; lse includes the offsets, so
    exp(lse) is the Horvitz-Thompson estimate of the softmax normaliser and exp(lse) * o that of
    its numerator.  A row with no kept block gives o = 0 and lse = -inf."""
    dec = bf16_bits_to_f64 if q.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    B, H, N, D = q.shape
    NB = N // blk
    o = np.zeros((B, H, N, D))
    lse = np.full((B, H, N), -np.inf)
    for b in range(B):
        for h in range(H):
            kh, vh = dec(k[b, h]), dec(v[b, h])
            for i in range(NB):
                kept = np.nonzero(keep[b, h, i])[0]
                if kept.size == 0:
                    continue
                if (pi[b, h, i, kept] <= 0).any():
                    raise ValueError("a kept block must have a positive inclusion probability")
                tok = (kept[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
                off = np.repeat(-np.log(pi[b, h, i, kept]), blk)
                rows = slice(i * blk, (i + 1) * blk)
                s = dec(q[b, h, rows]) @ kh[tok].T * scale + off[None, :]
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=1, keepdims=True)
                o[b, h, rows] = (e @ vh[tok]) / l
                lse[b, h, rows] = (m + np.log(l))[:, 0]
    return o, lse
