"""Shared helpers of the GPU parity tests (test code: conversions, packing and
the comparison rules; no method arithmetic)."""
from __future__ import annotations

import dataclasses
import math
from typing import List, Sequence, Tuple

import numpy as np
import torch

import dbst_synth as S
import oracle as O

# Correctness bounds for floating-point attention output (bf16 result vs the
# float64 oracle): element-wise max-abs error and relative L2 error.
ATTN_MAX_ABS = 2e-2
ATTN_REL_L2 = 5e-3
# log-sum-exp (natural log): fp32 logits of bf16 inputs, fp32 sums
LSE_MAX_ABS = 2e-3
# A kept/dropped disagreement is excused only where the oracle's cumulative
# pooled mass at that block's rank, or at the rank before it, lies within
# this distance of p.
CDF_EXEMPT = 1e-4


def bits_to_torch(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def torch_to_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().view(torch.int16).cpu().numpy().view(np.uint16)


def geometry(w: S.Workload, heads: int = None) -> O.Geometry:
    return O.Geometry(w.B, w.H if heads is None else heads, w.D, *w.grid, *w.tile)


def pack_mask(mask: np.ndarray) -> np.ndarray:
    """bool [..., NB] -> uint32 words [..., ceil(NB/32)], bit j%32 of word j//32."""
    nb = mask.shape[-1]
    nw = (nb + 31) // 32
    pad = np.zeros(mask.shape[:-1] + (nw * 32,), dtype=bool)
    pad[..., :nb] = mask
    by = np.packbits(pad, axis=-1, bitorder="little")
    return np.ascontiguousarray(by).view("<u4").reshape(mask.shape[:-1] + (nw,))


def unpack_mask(words: np.ndarray, nb: int) -> np.ndarray:
    by = np.ascontiguousarray(words.astype("<u4")).view(np.uint8)
    bits = np.unpackbits(by, axis=-1, bitorder="little")
    return bits[..., :nb].astype(bool)


def oracle_mask_per_head(qt: np.ndarray, kt: np.ndarray, g: O.Geometry, p: float, sta: int):
    """Oracle mask and reduced map, one (b, h) at a time to bound host memory."""
    B, H = qt.shape[0], qt.shape[1]
    mask = np.zeros((B, H, g.NB, g.NB), dtype=bool)
    A = np.zeros((B, H, g.NB, g.NB))
    g1 = dataclasses.replace(g, B=1, H=1)
    for b in range(B):
        for h in range(H):
            m, a = O.build_block_mask(qt[b:b + 1, h:h + 1], kt[b:b + 1, h:h + 1], g1, p, sta, return_scores=True)
            mask[b, h] = m[0, 0]
            A[b, h] = a[0, 0]
    return mask, A


def mask_mismatches(gpu: np.ndarray, ref: np.ndarray, A: np.ndarray, p: float, sta_mask: np.ndarray):
    """Non-excused disagreements between a GPU mask and the oracle mask.

    Returns (hard, excused): lists of (b, h, i, j).  Blocks forced by the
    sliding-tile neighbourhood must always agree.
    """
    hard, excused = [], []
    diff = np.argwhere(gpu != ref)
    for b, h, i, j in diff:
        if sta_mask[i, j] or p >= 1.0:
            hard.append((b, h, i, j))
            continue
        a = A[b, h, i]
        order = np.argsort(-a, kind="stable")
        c = np.cumsum(a[order])
        rank = int(np.nonzero(order == j)[0][0])            # 0-based
        near = abs(c[rank] - p) <= CDF_EXEMPT or (rank > 0 and abs(c[rank - 1] - p) <= CDF_EXEMPT)
        (excused if near else hard).append((int(b), int(h), int(i), int(j)))
    return hard, excused


def near_tie(A: np.ndarray, p: float, b: int, h: int, i: int, j: int, tol: float = 1e-6) -> bool:
    """Whether block j of row (b, h, i) ties (within `tol` in pooled mass) with the row's boundary
    block, the last one the oracle keeps.  Such disagreements are reported on their own; they are
    not excused."""
    a = A[b, h, i]
    order = np.argsort(-a, kind="stable")
    c = np.cumsum(a[order])
    k = min(int(np.searchsorted(c, p)), len(a) - 1) if p < 1.0 else len(a) - 1
    return abs(a[j] - a[order[k]]) <= tol


def write_mask_report(name: str, p: float, hard, excused, A: np.ndarray) -> None:
    """With DBST_PARITY_REPORT_DIR set, list every excused mask block (and every non-excused one,
    with its near-tie flag) in <dir>/mask_parity_<name>_p<p>.json."""
    import json
    import os
    out = os.environ.get("DBST_PARITY_REPORT_DIR")
    if not out:
        return
    os.makedirs(out, exist_ok=True)
    rep = {"workload": name, "p": p, "cdf_exemption": CDF_EXEMPT,
           "excused": [[int(x) for x in t] for t in excused],
           "not_excused": [[int(x) for x in t] + [bool(near_tie(A, p, *(int(x) for x in t)))] for t in hard]}
    with open(os.path.join(out, f"mask_parity_{name}_p{p}.json"), "w") as f:
        json.dump(rep, f)


def rows_where_masks_agree(got: np.ndarray, ref: np.ndarray, rows=None):
    """Query blocks (b, h, i) whose GPU mask row equals the oracle's row; from `rows`, or all.

    Attention parity feeds the oracle its own mask only.  A GPU output computed on the GPU's
    mask is therefore compared only where the two masks agree (they can differ only at
    near-threshold blocks, which the mask checks excuse)."""
    cand = rows if rows is not None else list(np.ndindex(*got.shape[:3]))
    return [tuple(int(x) for x in r) for r in cand if np.array_equal(got[tuple(r)], ref[tuple(r)])]


def lists_match_bits(cnt: np.ndarray, idx: np.ndarray, mask: np.ndarray) -> bool:
    if not np.array_equal(cnt, mask.sum(-1)):
        return False
    for pos in np.ndindex(*mask.shape[:-1]):
        js = np.nonzero(mask[pos])[0]
        if not np.array_equal(idx[pos][:js.size], js):
            return False
    return True


def attn_errors(o_gpu: np.ndarray, o_ref: np.ndarray) -> Tuple[float, float]:
    d = o_gpu.astype(np.float64) - o_ref
    max_abs = float(np.max(np.abs(d))) if d.size else 0.0
    den = float(np.linalg.norm(o_ref))
    rel = float(np.linalg.norm(d)) / den if den > 0 else float(np.linalg.norm(d))
    return max_abs, rel


def sample_rows(B: int, H: int, NB: int, count: int, seed: int) -> List[Tuple[int, int, int]]:
    rng = np.random.default_rng(seed)
    rows = {(0, 0, 0), (B - 1, H - 1, NB - 1)}
    while len(rows) < count:
        rows.add((int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(NB))))
    return sorted(rows)


def sample_rows_per_head(B: int, H: int, NB: int, per_head: int, seed: int) -> List[Tuple[int, int, int]]:
    """`per_head` distinct seeded query blocks in every (b, h), plus the first and the last block."""
    rng = np.random.default_rng(seed)
    rows = {(0, 0, 0), (B - 1, H - 1, NB - 1)}
    for b in range(B):
        for h in range(H):
            for i in rng.choice(NB, size=min(per_head, NB), replace=False):
                rows.add((b, h, int(i)))
    return sorted(rows)


def gpu_rows(t: torch.Tensor, rows: Sequence[Tuple[int, int, int]], blk: int = 64) -> np.ndarray:
    """Gather [len(rows), blk, ...] query blocks of a [B, H, N, ...] GPU tensor as float64."""
    out = [t[b, h, i * blk:(i + 1) * blk].float().cpu().numpy() for (b, h, i) in rows]
    return np.stack(out).astype(np.float64)
