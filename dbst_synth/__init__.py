"""Seeded synthetic Q/K/V shaped like latent video-DiT attention inputs.

This module is shared by the CPU oracle (``oracle/``), the GPU library's tests
and ``bench.py``.  It holds workload descriptions and random-number recipes
only; none of the attention method's arithmetic lives here.  Both sides of
every parity check consume the identical bf16 bit patterns produced below.

Recipe (per workload, per (batch, head) pair):

* ``rng = numpy.random.default_rng([seed, b, h])`` (PCG64, SeedSequence
  substreams), ``seed = 1000 + workload index``.
* A smooth field ``f_c(t, y, x) = sum_{m=1..4} sin(2*pi*(k_t t/T + k_y y/Y +
  k_x x/X) + phi_m)`` per channel ``c``; integer wave numbers
  ``k in {0..kmax}`` and phases ``phi ~ U[0, 2*pi)`` are drawn per (c, m).
  Each channel is normalised to RMS ``f_rms`` over the token grid.
* ``q = alpha * f + beta * eps_q``, ``k = alpha * f + beta * eps_k`` (the same
  ``f`` for both: the "Q=K basis"), ``v = eps_v``, with ``eps ~ N(0, 1)``.
* Values are rounded to bf16 with round-to-nearest-even on the host.
* The upstream gradient of the backward (``make_grad``) is ``N(0, 1)`` from
  ``default_rng([seed, b, h, 1])``, rounded the same way.

Tokens are laid out in raster order ``n = (t*Y + y)*X + x``, tensors are
``[B, H, N, D]`` contiguous.  The mixing weights ``alpha``/``beta`` follow the
workload descriptions; ``f_rms`` (the sinusoid amplitude) is not fixed by any
description and is chosen per workload so that the pooled-score map has the
concentration real DiT heads show (about 10 % of key blocks carry 90 % of the
pooled mass on the Wan-like shape).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import numpy as np

__all__ = ["Workload", "WORKLOADS", "workload", "make_qkv", "bf16_bits_from_f32",
           "f32_from_bf16_bits"]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                 # position in the workload list; seed = 1000 + index
    B: int
    H: int
    D: int
    grid: Tuple[int, int, int]   # token grid (T, Y, X)
    tile: Tuple[int, int, int]   # tile shape (tt, ty, tx); tt*ty*tx == 64
    alpha: float
    beta: float
    f_rms: float
    kmax: int
    p_list: Tuple[float, ...]
    sta_radius: int              # < 0: no sliding-tile neighbourhood
    unpadded: Optional[Tuple[int, int, int]] = None

    @property
    def N(self) -> int:
        T, Y, X = self.grid
        return T * Y * X

    @property
    def blk(self) -> int:
        return self.tile[0] * self.tile[1] * self.tile[2]

    @property
    def NB(self) -> int:
        return self.N // self.blk

    @property
    def tile_grid(self) -> Tuple[int, int, int]:
        return tuple(g // t for g, t in zip(self.grid, self.tile))

    @property
    def seed(self) -> int:
        return 1000 + self.index

    def tensor_bytes(self) -> int:
        return self.B * self.H * self.N * self.D * 2


WORKLOADS: List[Workload] = [
    Workload("tiny", 0, B=1, H=2, D=64, grid=(4, 8, 8), tile=(1, 8, 8),
             alpha=0.7, beta=0.3, f_rms=2.0, kmax=3, p_list=(0.9, 1.0), sta_radius=-1),
    Workload("small", 1, B=1, H=8, D=64, grid=(8, 16, 16), tile=(1, 8, 8),
             alpha=0.7, beta=0.3, f_rms=2.0, kmax=3, p_list=(0.8, 0.9, 0.95), sta_radius=1),
    Workload("wan", 2, B=1, H=40, D=128, grid=(21, 32, 56), tile=(1, 8, 8),
             alpha=0.5, beta=0.5, f_rms=2.54, kmax=3, p_list=(0.9,), sta_radius=-1,
             unpadded=(21, 30, 52)),
    Workload("hunyuan", 3, B=1, H=24, D=128, grid=(34, 48, 80), tile=(2, 4, 8),
             alpha=0.4, beta=0.6, f_rms=2.6, kmax=3, p_list=(0.9,), sta_radius=1,
             unpadded=(33, 45, 80)),
    Workload("sweep", 4, B=2, H=16, D=128, grid=(16, 32, 32), tile=(2, 4, 8),
             alpha=0.7, beta=0.3, f_rms=1.6, kmax=3,
             p_list=(0.5, 0.7, 0.8, 0.9, 0.95, 0.99, 1.0), sta_radius=-1),
    # The Wan-like latent in the 2x4x8 tiles its description names: 21 frames do not divide by 2,
    # so the grid is padded to 22 frames (11 x 8 x 7 tiles, 616 blocks).  f_rms is set, as for
    # "wan", so that p = 0.9 keeps about 10 % of blocks (9.9 %; the Wan value 2.54 keeps 0.4 % in
    # these tiles).
    Workload("wan_2x4x8", 5, B=1, H=40, D=128, grid=(22, 32, 56), tile=(2, 4, 8),
             alpha=0.5, beta=0.5, f_rms=2.23, kmax=3, p_list=(0.9,), sta_radius=-1,
             unpadded=(21, 30, 52)),
]


def workload(name: str) -> Workload:
    for w in WORKLOADS:
        if w.name == name:
            return w
    raise KeyError(name)


def bf16_bits_from_f32(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def f32_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _basis(grid: Tuple[int, int, int], kmax: int) -> np.ndarray:
    """sin/cos of every wave vector in {0..kmax}^3 over the raster grid.

    Returns float64 ``[2 * (kmax+1)^3, N]``: rows ``2w`` = sin, ``2w+1`` = cos
    of ``2*pi*(k_t t/T + k_y y/Y + k_x x/X)`` for wave vector index
    ``w = (k_t*(kmax+1) + k_y)*(kmax+1) + k_x``.
    """
    T, Y, X = grid
    t = np.arange(T, dtype=np.float64)[:, None, None]
    y = np.arange(Y, dtype=np.float64)[None, :, None]
    x = np.arange(X, dtype=np.float64)[None, None, :]
    K = kmax + 1
    rows = []
    for kt in range(K):
        for ky in range(K):
            for kx in range(K):
                theta = 2.0 * math.pi * (kt * t / T + ky * y / Y + kx * x / X)
                rows.append(np.sin(theta).reshape(-1))
                rows.append(np.cos(theta).reshape(-1))
    return np.stack(rows)


def _field(rng: np.random.Generator, D: int, kmax: int, basis: np.ndarray, f_rms: float) -> np.ndarray:
    """One head's smooth field ``f`` as float64 ``[N, D]`` with per-channel RMS ``f_rms``."""
    K3 = (kmax + 1) ** 3
    kidx = rng.integers(0, K3, size=(D, 4))
    phi = rng.uniform(0.0, 2.0 * math.pi, size=(D, 4))
    coef = np.zeros((D, 2 * K3), dtype=np.float64)
    # sin(theta + phi) = sin(theta) cos(phi) + cos(theta) sin(phi)
    for m in range(4):
        np.add.at(coef, (np.arange(D), 2 * kidx[:, m]), np.cos(phi[:, m]))
        np.add.at(coef, (np.arange(D), 2 * kidx[:, m] + 1), np.sin(phi[:, m]))
    f = coef @ basis                                   # [D, N]
    rms = np.sqrt(np.mean(f * f, axis=1, keepdims=True))
    rms[rms == 0.0] = 1.0
    return (f * (f_rms / rms)).T                       # [N, D]


def make_qkv(w: Workload, heads: Optional[range] = None, batches: Optional[range] = None):
    """Seeded q, k, v as bf16 bit patterns (``uint16``), raster order ``[B', H', N, D]``.

    ``heads``/``batches`` select a subset of (b, h) pairs; every pair's values
    depend only on (seed, b, h), so a subset equals the same slice of the full
    tensors.
    """
    heads = range(w.H) if heads is None else heads
    batches = range(w.B) if batches is None else batches
    basis = _basis(w.grid, w.kmax)
    shape = (len(batches), len(heads), w.N, w.D)
    q = np.empty(shape, np.uint16)
    k = np.empty(shape, np.uint16)
    v = np.empty(shape, np.uint16)
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            rng = np.random.default_rng([w.seed, b, h])
            f = _field(rng, w.D, w.kmax, basis, w.f_rms).astype(np.float32)
            eq = rng.standard_normal((w.N, w.D), dtype=np.float32)
            ek = rng.standard_normal((w.N, w.D), dtype=np.float32)
            ev = rng.standard_normal((w.N, w.D), dtype=np.float32)
            a = np.float32(w.alpha)
            be = np.float32(w.beta)
            q[bi, hi] = bf16_bits_from_f32(a * f + be * eq)
            k[bi, hi] = bf16_bits_from_f32(a * f + be * ek)
            v[bi, hi] = bf16_bits_from_f32(ev)
    return q, k, v


def make_grad(w: Workload, heads: Optional[range] = None, batches: Optional[range] = None) -> np.ndarray:
    """Seeded upstream gradient dO as bf16 bit patterns, raster order ``[B', H', N, D]``;
    per (b, h) it depends only on (seed, b, h), like :func:`make_qkv`."""
    heads = range(w.H) if heads is None else heads
    batches = range(w.B) if batches is None else batches
    out = np.empty((len(batches), len(heads), w.N, w.D), np.uint16)
    for bi, b in enumerate(batches):
        for hi, h in enumerate(heads):
            rng = np.random.default_rng([w.seed, b, h, 1])
            out[bi, hi] = bf16_bits_from_f32(rng.standard_normal((w.N, w.D), dtype=np.float32))
    return out
