"""Python binding of libdbst.so: block-sparse tile attention on B200 (sm_100a).

Argument marshalling only.  Every step of the path runs in the library's CUDA
kernels; there is no CPU or PyTorch fallback, and importing a function whose
library is missing raises immediately.  Tensors are torch CUDA tensors
(device memory and streams come from PyTorch); each call is enqueued on the
current torch stream.

Layouts follow ``include/dbst.h``: q, k, v, o are bf16 ``[B, H, N, D]``
contiguous, raster order ``n = (t*Y + y)*X + x`` or tile order.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence, Tuple

import torch

__all__ = ["Geom", "DbstError", "lib_path", "load", "tile_reorder", "tile_unreorder", "mask_workspace_bytes",
           "build_block_mask", "build_block_mask_noalloc", "mask_from_bits", "block_sparse_attn", "dense_attn",
           "build_block_mask_raster", "block_sparse_attn_raster", "dense_attn_raster", "pair_query_blocks",
           "transpose_block_mask", "attn_backward_workspace_bytes", "block_sparse_attn_backward",
           "squad_workspace_bytes", "squad_attn", "build_sip_mask", "block_sparse_attn_offsets",
           "fine_mask_workspace_bytes", "build_fine_mask", "block_sparse_attn_groups", "block_sparse_attn_gather",
           "get_error", "set_wait_limit", "EXPORTS"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdbst.so")

# Every symbol declared in include/dbst.h.
EXPORTS = ("dbst_status_string", "dbst_tile_reorder", "dbst_tile_unreorder", "dbst_mask_workspace_bytes",
           "dbst_build_block_mask", "dbst_mask_from_bits", "dbst_block_sparse_attn", "dbst_dense_attn",
           "dbst_get_error", "dbst_build_block_mask_noalloc", "dbst_build_block_mask_raster",
           "dbst_block_sparse_attn_raster", "dbst_dense_attn_raster", "dbst_pair_query_blocks",
           "dbst_transpose_block_mask", "dbst_attn_backward_workspace_bytes", "dbst_block_sparse_attn_backward",
           "dbst_block_sparse_attn_backward_raster", "dbst_squad_workspace_bytes", "dbst_squad_attn",
           "dbst_build_sip_mask", "dbst_build_sip_mask_raster", "dbst_block_sparse_attn_offsets",
           "dbst_block_sparse_attn_offsets_raster", "dbst_fine_mask_workspace_bytes", "dbst_build_fine_mask",
           "dbst_build_fine_mask_raster", "dbst_block_sparse_attn_groups", "dbst_block_sparse_attn_groups_raster",
           "dbst_block_sparse_attn_gather", "dbst_block_sparse_attn_gather_raster", "dbst_set_wait_limit",
           "dbst_block_sparse_attn_offsets_paired", "dbst_block_sparse_attn_offsets_paired_raster")

DBST_OK, DBST_EINVAL, DBST_ECUDA, DBST_ETIMEOUT, DBST_EBOUNDS, DBST_ETOOLARGE = 0, 1, 2, 3, 4, 5
NOALLOC_SCRATCH_BYTES = 64 << 20


class DbstError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {_status_string(status)} (status {status})")
        self.status = status


class Geom(ctypes.Structure):
    """Mirror of ``dbst_geom``: batch, heads, head dim, token grid, tile shape."""
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "D", "T", "Y", "X", "tt", "ty", "tx")]

    @classmethod
    def make(cls, B: int, H: int, D: int, grid: Sequence[int], tile: Sequence[int]) -> "Geom":
        return cls(B, H, D, *grid, *tile)

    @property
    def N(self) -> int:
        return self.T * self.Y * self.X

    @property
    def NB(self) -> int:
        return self.N // 64

    @property
    def NW(self) -> int:
        return (self.NB + 31) // 32


_lib = None


def lib_path() -> str:
    return _LIB_PATH


def load() -> ctypes.CDLL:
    """Load libdbst.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with `python -m dynamic_block_sparse_tile_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    vp, gp, i32, f32 = ctypes.c_void_p, ctypes.POINTER(Geom), ctypes.c_int, ctypes.c_float
    lib.dbst_status_string.argtypes, lib.dbst_status_string.restype = [i32], ctypes.c_char_p
    for name in ("dbst_tile_reorder", "dbst_tile_unreorder"):
        getattr(lib, name).argtypes = [vp, vp, gp, vp]
        getattr(lib, name).restype = i32
    lib.dbst_mask_workspace_bytes.argtypes, lib.dbst_mask_workspace_bytes.restype = [gp], ctypes.c_size_t
    for name in ("dbst_build_block_mask", "dbst_build_block_mask_raster"):
        getattr(lib, name).argtypes = [vp, vp, gp, f32, i32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        getattr(lib, name).restype = i32
    lib.dbst_mask_from_bits.argtypes, lib.dbst_mask_from_bits.restype = [vp, gp, vp, vp, vp], i32
    lib.dbst_block_sparse_attn.argtypes = [vp, vp, vp, gp, vp, vp, f32, vp, vp, vp]
    lib.dbst_block_sparse_attn.restype = i32
    lib.dbst_block_sparse_attn_raster.argtypes = [vp, vp, vp, gp, vp, vp, vp, f32, vp, vp, vp]
    lib.dbst_block_sparse_attn_raster.restype = i32
    lib.dbst_pair_query_blocks.argtypes, lib.dbst_pair_query_blocks.restype = [vp, gp, vp, vp], i32
    for name in ("dbst_dense_attn", "dbst_dense_attn_raster"):
        getattr(lib, name).argtypes, getattr(lib, name).restype = [vp, vp, vp, gp, f32, vp, vp, vp], i32
    lib.dbst_get_error.argtypes, lib.dbst_get_error.restype = [vp], i32
    lib.dbst_build_block_mask_noalloc.argtypes = [vp, vp, gp, f32, i32, vp, vp, vp, vp]
    lib.dbst_build_block_mask_noalloc.restype = i32
    lib.dbst_transpose_block_mask.argtypes, lib.dbst_transpose_block_mask.restype = [vp, gp, vp, vp, vp, vp], i32
    lib.dbst_attn_backward_workspace_bytes.argtypes = [gp]
    lib.dbst_attn_backward_workspace_bytes.restype = ctypes.c_size_t
    for name in ("dbst_block_sparse_attn_backward", "dbst_block_sparse_attn_backward_raster"):
        getattr(lib, name).argtypes = [vp, vp, vp, vp, vp, gp, vp, vp, vp, vp, f32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        getattr(lib, name).restype = i32
    lib.dbst_squad_workspace_bytes.argtypes = [i32, i32, i32, i32, i32]
    lib.dbst_squad_workspace_bytes.restype = ctypes.c_size_t
    lib.dbst_squad_attn.argtypes = [vp, vp, vp, i32, i32, i32, i32, i32, f32, vp, vp, ctypes.c_size_t, vp]
    lib.dbst_squad_attn.restype = i32
    for name in ("dbst_build_sip_mask", "dbst_build_sip_mask_raster"):
        getattr(lib, name).argtypes = [vp, vp, gp, ctypes.c_double, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, vp]
        getattr(lib, name).restype = i32
    for name in ("dbst_block_sparse_attn_offsets", "dbst_block_sparse_attn_offsets_raster"):
        getattr(lib, name).argtypes = [vp, vp, vp, gp, vp, vp, vp, f32, vp, vp, vp]
        getattr(lib, name).restype = i32
    for name in ("dbst_block_sparse_attn_offsets_paired", "dbst_block_sparse_attn_offsets_paired_raster"):
        getattr(lib, name).argtypes = [vp, vp, vp, gp, vp, vp, vp, vp, f32, vp, vp, vp]
        getattr(lib, name).restype = i32
    lib.dbst_fine_mask_workspace_bytes.argtypes = [gp]
    lib.dbst_fine_mask_workspace_bytes.restype = ctypes.c_size_t
    for name in ("dbst_build_fine_mask", "dbst_build_fine_mask_raster"):
        getattr(lib, name).argtypes = [vp, vp, gp, f32, vp, vp, vp, vp, ctypes.c_size_t, vp]
        getattr(lib, name).restype = i32
    for name in ("dbst_block_sparse_attn_gather", "dbst_block_sparse_attn_gather_raster"):
        getattr(lib, name).argtypes = [vp, vp, vp, gp, vp, f32, vp, vp, vp]
        getattr(lib, name).restype = i32
    for name in ("dbst_block_sparse_attn_groups", "dbst_block_sparse_attn_groups_raster"):
        getattr(lib, name).argtypes = [vp, vp, vp, gp, vp, vp, vp, f32, vp, vp, vp]
        getattr(lib, name).restype = i32
    lib.dbst_set_wait_limit.argtypes, lib.dbst_set_wait_limit.restype = [ctypes.c_longlong], None
    _lib = lib
    return lib


def _status_string(status: int) -> str:
    try:
        return load().dbst_status_string(status).decode()
    except Exception:
        return "unknown"


def _check(status: int, what: str) -> None:
    if status != DBST_OK:
        raise DbstError(status, what)


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> ctypes.c_void_p:
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _need(t: torch.Tensor, dtype: torch.dtype, shape: Tuple[int, ...], name: str) -> None:
    if not t.is_cuda or t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


def _qkv_shape(g: Geom) -> Tuple[int, int, int, int]:
    return (g.B, g.H, g.N, g.D)


def tile_reorder(x: torch.Tensor, g: Geom, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Raster -> tile order (``dbst_tile_reorder``)."""
    _need(x, torch.bfloat16, _qkv_shape(g), "x")
    out = torch.empty_like(x) if out is None else out
    _need(out, torch.bfloat16, _qkv_shape(g), "out")
    _check(load().dbst_tile_reorder(_ptr(x), _ptr(out), ctypes.byref(g), _stream()), "dbst_tile_reorder")
    return out


def tile_unreorder(y: torch.Tensor, g: Geom, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Tile -> raster order (``dbst_tile_unreorder``)."""
    _need(y, torch.bfloat16, _qkv_shape(g), "y")
    out = torch.empty_like(y) if out is None else out
    _need(out, torch.bfloat16, _qkv_shape(g), "out")
    _check(load().dbst_tile_unreorder(_ptr(y), _ptr(out), ctypes.byref(g), _stream()), "dbst_tile_unreorder")
    return out


def mask_workspace_bytes(g: Geom) -> int:
    return int(load().dbst_mask_workspace_bytes(ctypes.byref(g)))


def build_block_mask(q_tiled: torch.Tensor, k_tiled: torch.Tensor, g: Geom, p: float, sta_radius: int = -1,
                     workspace: Optional[torch.Tensor] = None, out=None):
    """Adaptive block mask (``dbst_build_block_mask``) -> (mask_bits, kv_count, kv_idx)."""
    return _build_block_mask("dbst_build_block_mask", q_tiled, k_tiled, g, p, sta_radius, workspace, out)


def build_block_mask_raster(q: torch.Tensor, k: torch.Tensor, g: Geom, p: float, sta_radius: int = -1,
                            workspace: Optional[torch.Tensor] = None, out=None):
    """Adaptive block mask from raster-order q, k (``dbst_build_block_mask_raster``)."""
    return _build_block_mask("dbst_build_block_mask_raster", q, k, g, p, sta_radius, workspace, out)


def _build_block_mask(fn: str, q_tiled, k_tiled, g: Geom, p: float, sta_radius: int, workspace, out):
    _need(q_tiled, torch.bfloat16, _qkv_shape(g), "q_tiled")
    _need(k_tiled, torch.bfloat16, _qkv_shape(g), "k_tiled")
    dev = q_tiled.device
    if out is None:
        bits = torch.empty((g.B, g.H, g.NB, g.NW), dtype=torch.int32, device=dev)
        cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device=dev)
        idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=dev)
    else:
        bits, cnt, idx = out
    nbytes = mask_workspace_bytes(g)
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    _check(getattr(load(), fn)(_ptr(q_tiled), _ptr(k_tiled), ctypes.byref(g), float(p), int(sta_radius),
                               _ptr(bits), _ptr(cnt), _ptr(idx), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream()), fn)
    return bits, cnt, idx


def build_block_mask_noalloc(q_tiled: torch.Tensor, k_tiled: torch.Tensor, g: Geom, p: float,
                             sta_radius: int = -1, out=None):
    """Adaptive block mask without a workspace argument (``dbst_build_block_mask_noalloc``).

    For callers that cannot allocate device memory: the library's fixed
    static scratch (``NOALLOC_SCRATCH_BYTES``) is used instead.  Output
    tensors are still the caller's (pass ``out`` to avoid allocating them here).
    """
    _need(q_tiled, torch.bfloat16, _qkv_shape(g), "q_tiled")
    _need(k_tiled, torch.bfloat16, _qkv_shape(g), "k_tiled")
    dev = q_tiled.device
    if out is None:
        bits = torch.empty((g.B, g.H, g.NB, g.NW), dtype=torch.int32, device=dev)
        cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device=dev)
        idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=dev)
    else:
        bits, cnt, idx = out
    _check(load().dbst_build_block_mask_noalloc(_ptr(q_tiled), _ptr(k_tiled), ctypes.byref(g), float(p),
                                                int(sta_radius), _ptr(bits), _ptr(cnt), _ptr(idx), _stream()),
           "dbst_build_block_mask_noalloc")
    return bits, cnt, idx


def mask_from_bits(bits: torch.Tensor, g: Geom):
    """Caller-supplied bitmask -> (kv_count, kv_idx) (``dbst_mask_from_bits``)."""
    _need(bits, torch.int32, (g.B, g.H, g.NB, g.NW), "bits")
    cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device=bits.device)
    idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=bits.device)
    _check(load().dbst_mask_from_bits(_ptr(bits), ctypes.byref(g), _ptr(cnt), _ptr(idx), _stream()),
           "dbst_mask_from_bits")
    return cnt, idx


def block_sparse_attn(q, k, v, g: Geom, kv_count, kv_idx, scale: float = 0.0, want_lse: bool = True,
                      out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None):
    """Attention over kept blocks (``dbst_block_sparse_attn``) -> (o, lse or None)."""
    return _block_sparse_attn("dbst_block_sparse_attn", q, k, v, g, kv_count, kv_idx, scale, want_lse, out, lse)


def block_sparse_attn_raster(q, k, v, g: Geom, kv_count, kv_idx, scale: float = 0.0, want_lse: bool = True,
                             out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                             pairs: Optional[torch.Tensor] = None):
    """Attention over kept blocks on raster-order tensors (``dbst_block_sparse_attn_raster``).

    ``pairs`` is an optional schedule from :func:`pair_query_blocks`.
    """
    if pairs is not None:
        _need(pairs, torch.int32, (g.B, g.H, (g.NB + 1) // 2), "pairs")
    return _block_sparse_attn("dbst_block_sparse_attn_raster", q, k, v, g, kv_count, kv_idx, scale, want_lse, out,
                              lse, pairs=pairs, with_pairs=True)


def pair_query_blocks(mask_bits: torch.Tensor, g: Geom, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Query-block pairs for the attention kernel (``dbst_pair_query_blocks``) -> int32 [B, H, ceil(NB/2)]."""
    _need(mask_bits, torch.int32, (g.B, g.H, g.NB, g.NW), "mask_bits")
    pairs = torch.empty((g.B, g.H, (g.NB + 1) // 2), dtype=torch.int32, device=mask_bits.device) if out is None else out
    _need(pairs, torch.int32, (g.B, g.H, (g.NB + 1) // 2), "pairs")
    _check(load().dbst_pair_query_blocks(_ptr(mask_bits), ctypes.byref(g), _ptr(pairs), _stream()),
           "dbst_pair_query_blocks")
    return pairs


def _block_sparse_attn(fn: str, q, k, v, g: Geom, kv_count, kv_idx, scale, want_lse, out, lse, pairs=None,
                       with_pairs=False):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, _qkv_shape(g), n)
    _need(kv_count, torch.int32, (g.B, g.H, g.NB), "kv_count")
    _need(kv_idx, torch.int16, (g.B, g.H, g.NB, g.NB), "kv_idx")
    o = torch.empty_like(q) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=q.device)
    lib = load()
    if with_pairs:
        _check(getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), _ptr(kv_count), _ptr(kv_idx), _ptr(pairs),
                                float(scale), _ptr(o), _ptr(lse if want_lse else None), _stream()), fn)
    else:
        _check(getattr(lib, fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), _ptr(kv_count), _ptr(kv_idx),
                                float(scale), _ptr(o), _ptr(lse if want_lse else None), _stream()), fn)
    return o, (lse if want_lse else None)


def dense_attn(q, k, v, g: Geom, scale: float = 0.0, want_lse: bool = True):
    """Dense attention over all tokens (``dbst_dense_attn``) -> (o, lse or None)."""
    return _dense_attn("dbst_dense_attn", q, k, v, g, scale, want_lse)


def dense_attn_raster(q, k, v, g: Geom, scale: float = 0.0, want_lse: bool = True):
    """Dense attention on raster-order tensors (``dbst_dense_attn_raster``) -> (o, lse or None)."""
    return _dense_attn("dbst_dense_attn_raster", q, k, v, g, scale, want_lse)


def _dense_attn(fn: str, q, k, v, g: Geom, scale, want_lse):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, _qkv_shape(g), n)
    o = torch.empty_like(q)
    lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=q.device) if want_lse else None
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), float(scale), _ptr(o), _ptr(lse),
                               _stream()), fn)
    return o, lse


def transpose_block_mask(mask_bits: torch.Tensor, g: Geom, out=None):
    """Transposed block mask and its lists (``dbst_transpose_block_mask``) -> (mask_bits_t, q_count, q_idx).

    Row j of the result lists the query blocks whose kept set contains key block j.
    """
    _need(mask_bits, torch.int32, (g.B, g.H, g.NB, g.NW), "mask_bits")
    dev = mask_bits.device
    if out is None:
        bits_t = torch.empty_like(mask_bits)
        cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device=dev)
        idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=dev)
    else:
        bits_t, cnt, idx = out
    _check(load().dbst_transpose_block_mask(_ptr(mask_bits), ctypes.byref(g), _ptr(bits_t), _ptr(cnt), _ptr(idx),
                                            _stream()), "dbst_transpose_block_mask")
    return bits_t, cnt, idx


def attn_backward_workspace_bytes(g: Geom) -> int:
    return int(load().dbst_attn_backward_workspace_bytes(ctypes.byref(g)))


def block_sparse_attn_backward(q, k, v, lse, d_o, g: Geom, kv_count, kv_idx, q_count, q_idx, scale: float = 0.0,
                               raster: bool = False, workspace: Optional[torch.Tensor] = None, out=None):
    """Gradients of the block-sparse attention (``dbst_block_sparse_attn_backward[_raster]``) -> (dq, dk, dv).

    ``lse`` is the forward's log-sum-exp for the same lists; (q_count, q_idx)
    come from :func:`transpose_block_mask` of the forward's mask.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (d_o, "d_o")):
        _need(t, torch.bfloat16, _qkv_shape(g), n)
    _need(lse, torch.float32, (g.B, g.H, g.N), "lse")
    for c, i, n in ((kv_count, kv_idx, "kv"), (q_count, q_idx, "q")):
        _need(c, torch.int32, (g.B, g.H, g.NB), f"{n}_count")
        _need(i, torch.int16, (g.B, g.H, g.NB, g.NB), f"{n}_idx")
    if out is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    else:
        dq, dk, dv = out
    if workspace is None:
        workspace = torch.empty(attn_backward_workspace_bytes(g), dtype=torch.uint8, device=q.device)
    fn = "dbst_block_sparse_attn_backward_raster" if raster else "dbst_block_sparse_attn_backward"
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), _ptr(v), _ptr(lse), _ptr(d_o), ctypes.byref(g), _ptr(kv_count),
                               _ptr(kv_idx), _ptr(q_count), _ptr(q_idx), float(scale), _ptr(dq), _ptr(dk), _ptr(dv),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream()), fn)
    return dq, dk, dv


def build_sip_mask(q, k, g: Geom, budget: float, uniforms: torch.Tensor, raster: bool = False,
                   workspace: Optional[torch.Tensor] = None, out=None):
    """Sampled block mask with inclusion-probability offsets (``dbst_build_sip_mask[_raster]``).

    ``uniforms``: float64 [B, H, NB, NB] in [0, 1).  Returns (mask_bits, kv_count, kv_idx, offsets),
    offsets float32 [B, H, NB, NB] = log(1/pi) at kept blocks.
    """
    _need(q, torch.bfloat16, _qkv_shape(g), "q")
    _need(k, torch.bfloat16, _qkv_shape(g), "k")
    _need(uniforms, torch.float64, (g.B, g.H, g.NB, g.NB), "uniforms")
    dev = q.device
    if out is None:
        bits = torch.empty((g.B, g.H, g.NB, g.NW), dtype=torch.int32, device=dev)
        cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device=dev)
        idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=dev)
        offsets = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.float32, device=dev)
    else:
        bits, cnt, idx, offsets = out
    if workspace is None:
        workspace = torch.empty(mask_workspace_bytes(g), dtype=torch.uint8, device=dev)
    fn = "dbst_build_sip_mask_raster" if raster else "dbst_build_sip_mask"
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), ctypes.byref(g), float(budget), _ptr(uniforms), _ptr(bits),
                               _ptr(cnt), _ptr(idx), _ptr(offsets), _ptr(workspace),
                               workspace.numel() * workspace.element_size(), _stream()), fn)
    return bits, cnt, idx, offsets


def block_sparse_attn_offsets(q, k, v, g: Geom, kv_count, kv_idx, offsets: Optional[torch.Tensor] = None,
                              scale: float = 0.0, raster: bool = False, want_lse: bool = True,
                              out: Optional[torch.Tensor] = None, lse: Optional[torch.Tensor] = None,
                              pairs: Optional[torch.Tensor] = None):
    """Attention over kept blocks with a logit offset per (query block, key block)
    (``dbst_block_sparse_attn_offsets[_raster]``, or ``..._offsets_paired[_raster]`` on the schedule
    ``pairs`` of :func:`pair_query_blocks`) -> (o, lse or None)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, _qkv_shape(g), n)
    _need(kv_count, torch.int32, (g.B, g.H, g.NB), "kv_count")
    _need(kv_idx, torch.int16, (g.B, g.H, g.NB, g.NB), "kv_idx")
    if offsets is not None:
        _need(offsets, torch.float32, (g.B, g.H, g.NB, g.NB), "offsets")
    o = torch.empty_like(q) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=q.device)
    if pairs is not None:
        _need(pairs, torch.int32, (g.B, g.H, (g.NB + 1) // 2), "pairs")
        fn = "dbst_block_sparse_attn_offsets_paired_raster" if raster else "dbst_block_sparse_attn_offsets_paired"
        _check(getattr(load(), fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), _ptr(kv_count), _ptr(kv_idx),
                                   _ptr(offsets), _ptr(pairs), float(scale), _ptr(o),
                                   _ptr(lse if want_lse else None), _stream()), fn)
        return o, (lse if want_lse else None)
    fn = "dbst_block_sparse_attn_offsets_raster" if raster else "dbst_block_sparse_attn_offsets"
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), _ptr(kv_count), _ptr(kv_idx),
                               _ptr(offsets), float(scale), _ptr(o), _ptr(lse if want_lse else None), _stream()), fn)
    return o, (lse if want_lse else None)


def fine_mask_workspace_bytes(g: Geom) -> int:
    return int(load().dbst_fine_mask_workspace_bytes(ctypes.byref(g)))


def build_fine_mask(q, k, g: Geom, p: float, raster: bool = False, workspace: Optional[torch.Tensor] = None,
                    out=None):
    """Mask of kept 4-token key groups (``dbst_build_fine_mask[_raster]``) -> (group_mask, kv_count, kv_idx).

    group_mask: int16 [B, H, NB, NB], bit r of [.., i, j] = group r (tokens 4r .. 4r+3) of key block j.
    """
    _need(q, torch.bfloat16, _qkv_shape(g), "q")
    _need(k, torch.bfloat16, _qkv_shape(g), "k")
    dev = q.device
    if out is None:
        gm = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=dev)
        cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device=dev)
        idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device=dev)
    else:
        gm, cnt, idx = out
    nbytes = fine_mask_workspace_bytes(g)
    if nbytes == 0:
        raise ValueError("fine mask: unsupported geometry (at most 1024 blocks per head)")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    fn = "dbst_build_fine_mask_raster" if raster else "dbst_build_fine_mask"
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), ctypes.byref(g), float(p), _ptr(gm), _ptr(cnt), _ptr(idx),
                               _ptr(workspace), workspace.numel() * workspace.element_size(), _stream()), fn)
    return gm, cnt, idx


def block_sparse_attn_groups(q, k, v, g: Geom, kv_count, kv_idx, group_mask, scale: float = 0.0,
                             raster: bool = False, want_lse: bool = True, out: Optional[torch.Tensor] = None,
                             lse: Optional[torch.Tensor] = None):
    """Attention over the kept 4-token key groups (``dbst_block_sparse_attn_groups[_raster]``) -> (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, _qkv_shape(g), n)
    _need(kv_count, torch.int32, (g.B, g.H, g.NB), "kv_count")
    _need(kv_idx, torch.int16, (g.B, g.H, g.NB, g.NB), "kv_idx")
    _need(group_mask, torch.int16, (g.B, g.H, g.NB, g.NB), "group_mask")
    o = torch.empty_like(q) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=q.device)
    fn = "dbst_block_sparse_attn_groups_raster" if raster else "dbst_block_sparse_attn_groups"
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), _ptr(kv_count), _ptr(kv_idx),
                               _ptr(group_mask), float(scale), _ptr(o), _ptr(lse if want_lse else None), _stream()), fn)
    return o, (lse if want_lse else None)


def block_sparse_attn_gather(q, k, v, g: Geom, group_mask, scale: float = 0.0, raster: bool = False,
                             want_lse: bool = True, out: Optional[torch.Tensor] = None,
                             lse: Optional[torch.Tensor] = None):
    """Attention over the kept 4-token key groups, gathered 16 to a tile
    (``dbst_block_sparse_attn_gather[_raster]``) -> (o, lse)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, _qkv_shape(g), n)
    _need(group_mask, torch.int16, (g.B, g.H, g.NB, g.NB), "group_mask")
    o = torch.empty_like(q) if out is None else out
    if want_lse and lse is None:
        lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device=q.device)
    fn = "dbst_block_sparse_attn_gather_raster" if raster else "dbst_block_sparse_attn_gather"
    _check(getattr(load(), fn)(_ptr(q), _ptr(k), _ptr(v), ctypes.byref(g), _ptr(group_mask), float(scale), _ptr(o),
                               _ptr(lse if want_lse else None), _stream()), fn)
    return o, (lse if want_lse else None)


def squad_workspace_bytes(B: int, H: int, N: int, D: int, w: int) -> int:
    return int(load().dbst_squad_workspace_bytes(B, H, N, D, w))


def squad_attn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, w: int, scale: float = 0.0,
               workspace: Optional[torch.Tensor] = None, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """SQuad two-pass attention with window w (``dbst_squad_attn``) on [B, H, N, D] bf16 -> o."""
    if q.dim() != 4:
        raise ValueError("q: expected [B, H, N, D]")
    B, H, N, D = q.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, (B, H, N, D), n)
    o = torch.empty_like(q) if out is None else out
    _need(o, torch.bfloat16, (B, H, N, D), "out")
    nbytes = squad_workspace_bytes(B, H, N, D, w)
    if nbytes == 0:
        raise ValueError(f"unsupported SQuad shape N={N} D={D} w={w}: w and N/w must be multiples of 64")
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    _check(load().dbst_squad_attn(_ptr(q), _ptr(k), _ptr(v), B, H, N, D, int(w), float(scale), _ptr(o),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(), _stream()),
           "dbst_squad_attn")
    return o


def get_error() -> None:
    """Synchronise the current stream and raise if a kernel recorded an error."""
    _check(load().dbst_get_error(_stream()), "device")


def set_wait_limit(cycles: int) -> None:
    """Limit (SM cycles) of the attention kernels' waits between roles (``dbst_set_wait_limit``); <= 0: default."""
    load().dbst_set_wait_limit(int(cycles))
