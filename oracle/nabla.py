"""fp64 oracle of the NABLA block-sparse attention path (test infrastructure).

Every function restates one step of the method described on the page
"NABLA: Neighborhood Adaptive Block-Level Attention", section "Méthodologie :
NABLA".  Inputs are bf16 bit patterns (``uint16``) or float arrays; all
arithmetic is float64.  Library primitives used as steps: ``numpy.matmul``,
``numpy.argsort`` (stable), ``numpy.cumsum``, ``numpy.exp``.

Readings adopted where the page is silent, ambiguous or garbled:

R1  CDF threshold ("Seuil CDF").  The page thresholds the row's cumulative
    probability at 1 - thr without fixing the sort direction.  Read with the
    row sorted ascending and cumulative mass c_j up to and including block j,
    block j is kept iff c_j > 1 - p.  Equivalently (and this is the form
    computed here): sort the row descending, ties to the lower key-block
    index first; C_k = sum of the k largest values; k* = min{k : C_k >= p};
    keep the k* largest.  With p >= 1 every block is kept.  The two forms
    select the same set except at exact ties and within rounding of p; a
    test checks that they agree on tie-free rows.
R2  Scale of the reduced map ("Attention Réduite").  Not stated; the
    pooled logits use the attention scale 1/sqrt(D).
R3  Ties in the sort: lower key-block index first.
R4  p must lie in (0, 1]; every row then keeps at least one block.
R5  A query block with no kept key block (only possible with a mask the
    caller supplies) produces output 0 and log-sum-exp -inf.
R6  Sliding-tile neighbourhood ("Intégration Hybride avec STA"; the lay
    section describes the own tile plus its direct neighbours):
    key tile j is a neighbour of query tile i iff the Chebyshev distance of
    their tile coordinates is <= r, clipped at the grid edges (no wrap, no
    shifting of the window).
R7  Token reorder ("Fractal Flattening") generalised from P x P spatial
    patches to t x y x x tiles: tiles in raster order of tile coordinates,
    tokens inside a tile in raster order.  The time order of tiles is kept.
R8  Blocks are the 64-token tiles: the pooling block of N tokens is one
    tile, so query block i and key block j both mean tile i / tile j.
R9  Backward (the page claims faster training, sections "Contributions Clés"
    and "Résultats Expérimentaux", but prints no backward): the
    exact gradient of the forward definition of :func:`masked_attention`
    with respect to q, k and v, for an upstream gradient do of o.  A key
    token receives gradient only from the query blocks that keep its block;
    a query block with no kept key block receives none.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence, Tuple

import numpy as np


@dataclasses.dataclass(frozen=True)
class Geometry:
    """Shape of one call: batch, heads, head dim, token grid and tile shape."""
    B: int
    H: int
    D: int
    T: int
    Y: int
    X: int
    tt: int
    ty: int
    tx: int

    @property
    def N(self) -> int:
        return self.T * self.Y * self.X

    @property
    def blk(self) -> int:
        return self.tt * self.ty * self.tx

    @property
    def NB(self) -> int:
        return self.N // self.blk

    @property
    def tile_grid(self) -> Tuple[int, int, int]:
        return (self.T // self.tt, self.Y // self.ty, self.X // self.tx)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns: the bf16 value is the top half of an IEEE float32."""
    u32 = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u32.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Token reorder: "Réordonnancement des Jetons (Fractal Flattening)"
# ---------------------------------------------------------------------------

def tile_reorder(x: np.ndarray, g: Geometry) -> np.ndarray:
    """Raster token order -> tile order (reading R7).

    ``x`` is ``[B, H, N, D]`` with token n = (t*Y + y)*X + x.  In the result,
    token (t, y, x) sits at position
    ``((Tt*nY + Ty)*nX + Tx)*blk + (dt*ty + dy)*tx + dx`` where
    ``Tt, dt = divmod(t, tt)`` etc.  Any dtype; the copy is exact.
    """
    nT, nY, nX = g.tile_grid
    B, H = x.shape[0], x.shape[1]
    v = x.reshape(B, H, nT, g.tt, nY, g.ty, nX, g.tx, -1)
    # axes: B H Tt dt Ty dy Tx dx D  ->  B H Tt Ty Tx dt dy dx D
    v = v.transpose(0, 1, 2, 4, 6, 3, 5, 7, 8)
    return np.ascontiguousarray(v).reshape(B, H, g.N, -1)


def tile_unreorder(y: np.ndarray, g: Geometry) -> np.ndarray:
    """Tile order -> raster order; the inverse of :func:`tile_reorder`."""
    nT, nY, nX = g.tile_grid
    B, H = y.shape[0], y.shape[1]
    v = y.reshape(B, H, nT, nY, nX, g.tt, g.ty, g.tx, -1)
    # axes: B H Tt Ty Tx dt dy dx D  ->  B H Tt dt Ty dy Tx dx D
    v = v.transpose(0, 1, 2, 5, 3, 6, 4, 7, 8)
    return np.ascontiguousarray(v).reshape(B, H, g.N, -1)


# ---------------------------------------------------------------------------
# Adaptive mask: "Sous-échantillonnage", "Attention Réduite", "Seuil CDF"
# ---------------------------------------------------------------------------

def block_mean_pool(x_tiled: np.ndarray, blk: int) -> np.ndarray:
    """Mean of each run of ``blk`` consecutive tiled tokens, fp64 ``[B, H, NB, D]``."""
    x = np.asarray(x_tiled, dtype=np.float64)
    B, H, N, D = x.shape
    return x.reshape(B, H, N // blk, blk, D).sum(axis=3) / blk


def pooled_score_map(qp: np.ndarray, kp: np.ndarray, scale: float) -> np.ndarray:
    """Softmax over key blocks of the pooled logits (reading R2).

    ``A[b,h,i,j] = exp(s_ij - max_j s_ij) / sum_j exp(s_ij - max_j s_ij)``
    with ``s_ij = scale * <qp_i, kp_j>``.
    """
    s = np.matmul(qp, np.swapaxes(kp, -1, -2)) * scale
    s = s - s.max(axis=-1, keepdims=True)
    e = np.exp(s)
    return e / e.sum(axis=-1, keepdims=True)


def cdf_select_row(a: np.ndarray, p: float) -> np.ndarray:
    """Boolean keep-vector for one row of the reduced map (readings R1, R3).

    Sort descending with ties to the lower index, take the shortest prefix
    whose cumulative mass reaches ``p``.
    """
    nb = a.shape[0]
    keep = np.zeros(nb, dtype=bool)
    if p >= 1.0:
        keep[:] = True
        return keep
    order = np.argsort(-a, kind="stable")      # descending; stable => lower index first on ties
    c = np.cumsum(a[order])
    reached = np.nonzero(c >= p)[0]
    kstar = int(reached[0]) + 1 if reached.size else nb
    keep[order[:kstar]] = True
    return keep


def cdf_select(A: np.ndarray, p: float) -> np.ndarray:
    """:func:`cdf_select_row` applied to every row of ``A[..., NB, NB]``."""
    flat = A.reshape(-1, A.shape[-1])
    out = np.stack([cdf_select_row(r, p) for r in flat])
    return out.reshape(A.shape)


# ---------------------------------------------------------------------------
# "Intégration Hybride avec STA": M = M_nabla OR M_STA
# ---------------------------------------------------------------------------

def sta_mask(g: Geometry, radius: int) -> np.ndarray:
    """Block-level sliding-tile neighbourhood ``[NB, NB]`` (reading R6)."""
    nT, nY, nX = g.tile_grid
    NB = nT * nY * nX
    if radius < 0:
        return np.zeros((NB, NB), dtype=bool)
    idx = np.arange(NB)
    ct, rem = np.divmod(idx, nY * nX)
    cy, cx = np.divmod(rem, nX)
    dist = np.maximum(np.maximum(np.abs(ct[:, None] - ct[None, :]),
                                 np.abs(cy[:, None] - cy[None, :])),
                      np.abs(cx[:, None] - cx[None, :]))
    return dist <= radius


def build_block_mask(q_tiled: np.ndarray, k_tiled: np.ndarray, g: Geometry, p: float,
                     sta_radius: int = -1, scale: Optional[float] = None,
                     return_scores: bool = False):
    """Full mask construction: pool -> reduced map -> CDF select -> OR STA.

    ``q_tiled``/``k_tiled`` are tile-ordered (bf16 bits or floats).  Returns a
    boolean ``[B, H, NB, NB]`` block mask (and the reduced map if asked).
    """
    if not (0.0 < p <= 1.0):
        raise ValueError("p must lie in (0, 1]")
    if q_tiled.dtype == np.uint16:
        q_tiled = bf16_bits_to_f64(q_tiled)
        k_tiled = bf16_bits_to_f64(k_tiled)
    scale = 1.0 / math.sqrt(g.D) if scale is None else scale
    qp = block_mean_pool(q_tiled, g.blk)
    kp = block_mean_pool(k_tiled, g.blk)
    A = pooled_score_map(qp, kp, scale)
    mask = cdf_select(A, p) | sta_mask(g, sta_radius)[None, None]
    return (mask, A) if return_scores else mask


def mask_to_lists(mask: np.ndarray):
    """Expansion to per-query-block index lists (ascending key-block order).

    Returns ``kv_count [B, H, NB]`` int32 and ``kv_idx [B, H, NB, NB]`` int16
    where entries past ``kv_count`` are unspecified (filled with -1 here).
    """
    B, H, NB, _ = mask.shape
    count = mask.sum(axis=-1).astype(np.int32)
    idx = np.full((B, H, NB, NB), -1, dtype=np.int16)
    for b in range(B):
        for h in range(H):
            for i in range(NB):
                js = np.nonzero(mask[b, h, i])[0]
                idx[b, h, i, :js.size] = js
    return count, idx


# ---------------------------------------------------------------------------
# "Expansion": exact softmax attention over the tokens of the kept blocks
# ---------------------------------------------------------------------------

def masked_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, blk: int,
                     scale: float, rows: Optional[Sequence[Tuple[int, int, int]]] = None):
    """Attention of each query block over the tokens of its kept key blocks.

    ``q, k, v``: tile-ordered ``[B, H, N, D]`` (bf16 bits or floats).
    ``mask``: boolean ``[B, H, NB, NB]``.  For query token n in block i,
    ``o_n = sum_{m in S_i} softmax_m(scale * <q_n, k_m>) v_m`` with
    ``S_i`` the tokens of the kept key blocks of row i; ``lse_n`` is the
    natural-log log-sum-exp of the scaled logits.  Reading R5 for empty rows.

    ``rows``: optional list of (b, h, i) query blocks to compute; the result
    then holds only those blocks, shape ``[len(rows), blk, D]`` /
    ``[len(rows), blk]``.  Otherwise the full ``[B, H, N, D]`` / ``[B, H, N]``.
    """
    # bf16 inputs are decoded one query block / key set at a time (bounded host memory)
    dec = bf16_bits_to_f64 if q.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    B, H, N, D = q.shape
    NB = N // blk
    full = rows is None
    if full:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(NB)]
    o_out = np.zeros((len(rows), blk, D))
    lse_out = np.full((len(rows), blk), -np.inf)
    for r, (b, h, i) in enumerate(rows):
        kept = np.nonzero(mask[b, h, i])[0]
        if kept.size == 0:
            continue
        tok = (kept[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
        qi = dec(q[b, h, i * blk:(i + 1) * blk])
        ks = dec(k[b, h, tok])
        vs = dec(v[b, h, tok])
        s = (qi @ ks.T) * scale
        mx = s.max(axis=1, keepdims=True)
        e = np.exp(s - mx)
        den = e.sum(axis=1, keepdims=True)
        o_out[r] = (e @ vs) / den
        lse_out[r] = (mx + np.log(den))[:, 0]
    if full:
        return o_out.reshape(B, H, N, D), lse_out.reshape(B, H, N)
    return o_out, lse_out


def masked_attention_backward(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, blk: int,
                              scale: float, do: np.ndarray):
    """Gradients (dq, dk, dv) of :func:`masked_attention` for upstream gradient ``do`` (reading R9).

    Per query block i with kept key tokens S_i, with P the row softmax of
    s = scale * q_i k_S^T and o_i = P v_S (the softmax calculus, step by step):
        dv_S += P^T do_i,  dP = do_i v_S^T,  delta = rowsum(do_i * o_i),
        ds = P * (dP - delta),  dq_i = scale * ds k_S,  dk_S += scale * ds^T q_i.
    All inputs ``[B, H, N, D]`` tile-ordered (bf16 bits or floats); float64 out.
    """
    dec = bf16_bits_to_f64 if q.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    B, H, N, D = q.shape
    NB = N // blk
    do = np.asarray(do, dtype=np.float64)
    dq = np.zeros((B, H, N, D))
    dk = np.zeros((B, H, N, D))
    dv = np.zeros((B, H, N, D))
    for b in range(B):
        for h in range(H):
            kh, vh = dec(k[b, h]), dec(v[b, h])
            for i in range(NB):
                kept = np.nonzero(mask[b, h, i])[0]
                if kept.size == 0:
                    continue
                tok = (kept[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
                rows = slice(i * blk, (i + 1) * blk)
                qi, ks, vs, doi = dec(q[b, h, rows]), kh[tok], vh[tok], do[b, h, rows]
                s = (qi @ ks.T) * scale
                e = np.exp(s - s.max(axis=1, keepdims=True))
                P = e / e.sum(axis=1, keepdims=True)
                oi = P @ vs
                dv[b, h, tok] += P.T @ doi
                dP = doi @ vs.T
                delta = np.sum(doi * oi, axis=1, keepdims=True)
                ds = P * (dP - delta)
                dq[b, h, rows] = scale * (ds @ ks)
                dk[b, h, tok] += scale * (ds.T @ qi)
    return dq, dk, dv


def masked_attention_backward_blocks(q: np.ndarray, k: np.ndarray, v: np.ndarray, mask: np.ndarray, blk: int,
                                     scale: float, do: np.ndarray, q_blocks, k_blocks):
    """The gradients of :func:`masked_attention_backward` for chosen blocks only (reading R9).

    ``q_blocks``: iterable of (b, h, i) -> dq of query block i, ``[blk, D]``.
    ``k_blocks``: iterable of (b, h, j) -> (dk, dv) of key block j, each ``[blk, D]``; they sum
    over every query block that keeps j, so each such row is computed in full.
    Returns two dicts keyed by those tuples.  Same arithmetic as the full function, restricted.
    """
    dec = bf16_bits_to_f64 if q.dtype == np.uint16 else (lambda a: np.asarray(a, dtype=np.float64))
    q_blocks = [tuple(int(x) for x in t) for t in q_blocks]
    k_blocks = [tuple(int(x) for x in t) for t in k_blocks]
    want_q = set(q_blocks)
    want_k = {}
    for b, h, j in k_blocks:
        want_k.setdefault((b, h), set()).add(j)
    D = q.shape[-1]
    dq_out = {}
    dkv = {t: (np.zeros((blk, D)), np.zeros((blk, D))) for t in k_blocks}
    heads = {(b, h) for b, h, _ in q_blocks} | set(want_k)
    for b, h in sorted(heads):
        kj = want_k.get((b, h), set())
        rows = {i for bb, hh, i in q_blocks if (bb, hh) == (b, h)}
        for j in kj:
            rows |= set(np.nonzero(mask[b, h, :, j])[0].tolist())
        for i in sorted(rows):
            kept = np.nonzero(mask[b, h, i])[0]
            if kept.size == 0:
                if (b, h, i) in want_q:
                    dq_out[(b, h, i)] = np.zeros((blk, D))
                continue
            tok = (kept[:, None] * blk + np.arange(blk)[None, :]).reshape(-1)
            r = slice(i * blk, (i + 1) * blk)
            qi, ks, vs = dec(q[b, h, r]), dec(k[b, h, tok]), dec(v[b, h, tok])
            doi = np.asarray(do[b, h, r], dtype=np.float64)
            s = (qi @ ks.T) * scale
            e = np.exp(s - s.max(axis=1, keepdims=True))
            P = e / e.sum(axis=1, keepdims=True)
            oi = P @ vs
            dP = doi @ vs.T
            delta = np.sum(doi * oi, axis=1, keepdims=True)
            ds = P * (dP - delta)
            if (b, h, i) in want_q:
                dq_out[(b, h, i)] = scale * (ds @ ks)
            for pos, j in enumerate(kept):
                if int(j) in kj:
                    c = slice(pos * blk, (pos + 1) * blk)
                    dk_j, dv_j = dkv[(b, h, int(j))]
                    dk_j += scale * (ds[:, c].T @ qi)
                    dv_j += P[:, c].T @ doi
    for t in q_blocks:
        dq_out.setdefault(t, np.zeros((blk, D)))
    return dq_out, dkv


def dense_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """softmax(scale * q k^T) v over all tokens, fp64; returns (o, lse)."""
    if q.dtype == np.uint16:
        q, k, v = bf16_bits_to_f64(q), bf16_bits_to_f64(k), bf16_bits_to_f64(v)
    s = np.matmul(q, np.swapaxes(k, -1, -2)) * scale
    mx = s.max(axis=-1, keepdims=True)
    e = np.exp(s - mx)
    den = e.sum(axis=-1, keepdims=True)
    return np.matmul(e, v) / den, (mx + np.log(den))[..., 0]


def kept_pair_flops(kv_count: np.ndarray, D: int, blk: int = 64) -> float:
    """FLOPs of attention restricted to kept block pairs: 4 * D * blk^2 per pair."""
    return 4.0 * D * blk * blk * float(np.sum(kv_count, dtype=np.int64))
