"""Float64 oracle of fine-grained key selection: key groups of a few tokens.

TEST INFRASTRUCTURE ONLY (see the package docstring): nothing in the library
imports it.

Source: "AB-Attention accélère la génération vidéo jusqu'à 2,23× en sautant 92%
de l'attention" (news.hamidun.com), section "Les trois techniques", third
technique: key/value blocks of only 4 tokens, selected by index and gathered
by the kernel into full-size tensor-core tiles, without permuting tokens; at a
fixed tile budget, 4-token blocks keep more attention mass than 128-token ones.

Readings where the page is silent:

F1  Scoring and selection follow the NABLA path of ``oracle.nabla`` with a
    finer key unit: each 64-token query block is mean-pooled as before, each
    run of G consecutive tile-ordered key tokens ("group") is mean-pooled, the
    pooled logits (scale 1/sqrt(D)) are soft-maxed over all groups of the row,
    and the row keeps the smallest descending prefix of groups whose mass
    reaches p (``cdf_select_row``, ties to the lower index).  AB-Attention's own
    scorer (IBCS) is out of scope.
F2  G = 4 (the page's size); G must divide 64, so a group never straddles two
    tiles, and G = 64 is exactly the NABLA block mask.
F3  The gather order is free: the result is attention over the union of the
    kept groups' tokens, whatever order a kernel assembles them in.
"""
from __future__ import annotations

import numpy as np

from .nabla import Geometry, bf16_bits_to_f64, block_mean_pool, cdf_select, pooled_score_map


def fine_score_map(q_tiled: np.ndarray, k_tiled: np.ndarray, g: Geometry, G: int, scale=None) -> np.ndarray:
    """Pooled map ``[B, H, NB, N/G]``: softmax over key groups of <mean q block, mean k group>."""
    if G < 1 or 64 % G:
        raise ValueError("the group size must divide 64")
    dec = bf16_bits_to_f64 if q_tiled.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    qp = block_mean_pool(dec(q_tiled), g.blk)
    kp = block_mean_pool(dec(k_tiled), G)
    return pooled_score_map(qp, kp, (1.0 / np.sqrt(g.D)) if scale is None else scale)


def build_fine_mask(q_tiled: np.ndarray, k_tiled: np.ndarray, g: Geometry, p: float, G: int = 4,
                    return_scores: bool = False):
    """Kept key groups per query block, boolean ``[B, H, NB, N/G]`` (reading F1)."""
    if not (0.0 < p <= 1.0):
        raise ValueError("p must lie in (0, 1]")
    A = fine_score_map(q_tiled, k_tiled, g, G)
    mask = cdf_select(A, p)
    return (mask, A) if return_scores else mask


def fine_masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, blk: int, G: int,
                          scale: float):
    """Attention of each ``blk``-row query block over the tokens of its kept key groups.

    q, k, v ``[B, H, N, D]`` tile-ordered (bf16 bits or floats), mask ``[B, H, N/blk, N/G]``.
    Returns (o, lse) float64; a row with no kept group gives o = 0, lse = -inf.
    """
    dec = bf16_bits_to_f64 if q.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    B, H, N, D = q.shape
    o = np.zeros((B, H, N, D))
    lse = np.full((B, H, N), -np.inf)
    for b in range(B):
        for h in range(H):
            kh, vh = dec(k[b, h]), dec(v[b, h])
            for i in range(N // blk):
                kept = np.nonzero(mask[b, h, i])[0]
                if kept.size == 0:
                    continue
                tok = (kept[:, None] * G + np.arange(G)[None, :]).reshape(-1)
                rows = slice(i * blk, (i + 1) * blk)
                s = dec(q[b, h, rows]) @ kh[tok].T * scale
                m = s.max(axis=1, keepdims=True)
                e = np.exp(s - m)
                l = e.sum(axis=1, keepdims=True)
                o[b, h, rows] = (e @ vh[tok]) / l
                lse[b, h, rows] = (m + np.log(l))[:, 0]
    return o, lse


def kept_mass(A: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Pooled mass a mask keeps per row (the page's comparison of 4- and 128-token units)."""
    return np.where(mask, A, 0.0).sum(axis=-1)
