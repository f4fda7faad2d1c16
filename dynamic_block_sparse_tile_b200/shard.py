"""Head-parallel split of the path over ranks (one process per GPU).

Every (b, h) head is independent through the whole path: the block means, the
pooled score map, its CDF selection and the attention over the kept blocks are
each computed within one head (NABLA page, section "Méthodologie : NABLA").  A
job of H heads therefore runs on W GPUs as W independent calls, rank r taking
the contiguous heads ``head_range(H, W, r)``, with no collective on the data
path.  Only reassembling o on every rank needs one all-gather, done here with
``torch.distributed`` (NCCL between GPUs, gloo on CPU).

A caller whose activations are split by sequence instead (a DiT with
sequence parallelism) converts them to this head split with one all-to-all
before the path and back after it; that exchange belongs to the caller.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple

import torch

from . import (Geom, block_sparse_attn_raster, build_block_mask_raster, get_error, pair_query_blocks)

__all__ = ["head_range", "head_geometry", "local_heads", "run_local", "gather_heads", "run_sharded"]


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Heads [h0, h1) of rank ``rank``: contiguous, sizes differing by at most one (the first H % world ranks
    take one more)."""
    if world < 1 or not 0 <= rank < world or H < 1:
        raise ValueError(f"bad split: H={H} world={world} rank={rank}")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def head_geometry(g: Geom, h0: int, h1: int) -> Geom:
    """The same call geometry restricted to heads [h0, h1)."""
    return Geom.make(g.B, h1 - h0, g.D, (g.T, g.Y, g.X), (g.tt, g.ty, g.tx))


def local_heads(x: torch.Tensor, h0: int, h1: int) -> torch.Tensor:
    """Heads [h0, h1) of a [B, H, ...] tensor as a contiguous tensor."""
    return x[:, h0:h1].contiguous()


def run_local(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geom, p: float,
              sta_radius: int = -1) -> Tuple[torch.Tensor, torch.Tensor]:
    """The fused path on this rank's heads (raster q, k, v of geometry ``g``): mask, pair schedule, attention.
    Returns raster (o, lse).  No collective."""
    bits, cnt, idx = build_block_mask_raster(q, k, g, p, sta_radius)
    pairs = pair_query_blocks(bits, g)
    o, lse = block_sparse_attn_raster(q, k, v, g, cnt, idx, pairs=pairs)
    get_error()
    return o, lse


def gather_heads(local: torch.Tensor, H: int, world: int, rank: int, group=None) -> torch.Tensor:
    """All-gather of every rank's heads [h0, h1) of a [B, h1 - h0, ...] tensor into the full [B, H, ...] tensor.
    Ranks with one head fewer pad their share for the collective."""
    import torch.distributed as dist

    h0, h1 = head_range(H, world, rank)
    if local.shape[1] != h1 - h0:
        raise ValueError(f"rank {rank} holds {local.shape[1]} heads, its range is [{h0}, {h1})")
    hmax = head_range(H, world, 0)[1]
    send = local
    if local.shape[1] < hmax:
        pad = torch.zeros((local.shape[0], hmax - local.shape[1]) + tuple(local.shape[2:]), dtype=local.dtype,
                          device=local.device)
        send = torch.cat([local, pad], dim=1)
    send = send.contiguous()
    # bf16 travels as its 16-bit pattern: every backend moves int16
    as_bits = send.dtype == torch.bfloat16
    if as_bits:
        send = send.view(torch.int16)
    parts = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(parts, send, group=group)
    pieces = []
    for r in range(world):
        a, b = head_range(H, world, r)
        pieces.append(parts[r][:, :b - a])
    out = torch.cat(pieces, dim=1)
    return out.view(torch.bfloat16) if as_bits else out


def run_sharded(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: Geom, p: float, world: int, rank: int,
                sta_radius: int = -1, gather: bool = True, group=None,
                local_fn: Optional[Callable] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Rank ``rank`` of ``world`` runs the path on its heads of the full raster q, k, v (geometry ``g``) and, with
    ``gather``, reassembles the full o and lse on every rank.  ``local_fn(q, k, v, g_local, p, sta_radius)`` replaces
    the per-rank computation (``run_local``, the CUDA path) only where a test exercises the split itself."""
    h0, h1 = head_range(g.H, world, rank)
    gl = head_geometry(g, h0, h1)
    fn = run_local if local_fn is None else local_fn
    o, lse = fn(local_heads(q, h0, h1), local_heads(k, h0, h1), local_heads(v, h0, h1), gl, p, sta_radius)
    if not gather:
        return o, lse
    return gather_heads(o, g.H, world, rank, group), gather_heads(lse, g.H, world, rank, group)
