"""Host-side checks of the C ABI: the library loads, exports every declared
symbol, and rejects bad arguments before touching the GPU (no device needed)."""
import ctypes
import math
import os
import re

import pytest

import dynamic_block_sparse_tile_b200 as dbst
from dynamic_block_sparse_tile_b200 import build as dbst_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    dbst_build.build()
    return dbst.load()


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "dbst.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(dbst_[a-z_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_symbols()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(dbst.EXPORTS) == names


def test_status_strings(lib):
    assert lib.dbst_status_string(0) == b"ok"
    assert b"invalid" in lib.dbst_status_string(1)
    assert lib.dbst_status_string(99) == b"unknown status"


GOOD = dict(B=1, H=2, D=128, grid=(4, 8, 16), tile=(2, 4, 8))


def geom(**kw):
    a = dict(GOOD)
    a.update(kw)
    return dbst.Geom.make(a["B"], a["H"], a["D"], a["grid"], a["tile"])


BAD_GEOMS = [
    dict(D=96), dict(D=256), dict(B=0), dict(H=-1),
    dict(tile=(2, 4, 4)),                    # 32 tokens per tile
    dict(grid=(3, 8, 16)),                   # 3 frames not divisible by tt=2
    dict(grid=(4, 8, 12)),                   # 12 not divisible by tx=8
    dict(grid=(2, 512, 512), tile=(1, 8, 8)),  # NB = 8192 > 4096
]


@pytest.mark.parametrize("bad", BAD_GEOMS)
def test_bad_geometry_is_rejected_synchronously(lib, bad):
    g = geom(**bad)
    p = ctypes.c_void_p(1 << 20)
    assert lib.dbst_tile_reorder(p, ctypes.c_void_p(1 << 30), ctypes.byref(g), None) == dbst.DBST_EINVAL
    assert lib.dbst_mask_workspace_bytes(ctypes.byref(g)) == 0
    assert lib.dbst_dense_attn(p, p, p, ctypes.byref(g), 0.0, p, None, None) == dbst.DBST_EINVAL
    assert lib.dbst_mask_from_bits(p, ctypes.byref(g), p, p, None) == dbst.DBST_EINVAL


def test_null_and_misaligned_pointers(lib):
    g = geom()
    a, b = ctypes.c_void_p(1 << 20), ctypes.c_void_p(1 << 30)
    assert lib.dbst_tile_reorder(None, b, ctypes.byref(g), None) == dbst.DBST_EINVAL
    assert lib.dbst_tile_reorder(ctypes.c_void_p((1 << 20) + 8), b, ctypes.byref(g), None) == dbst.DBST_EINVAL
    assert lib.dbst_tile_reorder(a, a, ctypes.byref(g), None) == dbst.DBST_EINVAL           # in place
    assert lib.dbst_tile_unreorder(a, ctypes.c_void_p((1 << 20) + 64), ctypes.byref(g), None) == dbst.DBST_EINVAL
    assert lib.dbst_block_sparse_attn(a, a, a, ctypes.byref(g), None, a, 0.0, a, None, None) == dbst.DBST_EINVAL
    assert lib.dbst_block_sparse_attn(a, a, a, ctypes.byref(g), a, a, 0.0, a,
                                      ctypes.c_void_p((1 << 20) + 2), None) == dbst.DBST_EINVAL
    assert lib.dbst_dense_attn(a, a, a, ctypes.byref(g), float("nan"), a, None, None) == dbst.DBST_EINVAL
    assert lib.dbst_tile_reorder(a, b, None, None) == dbst.DBST_EINVAL
    # the raster entry points validate exactly like the tiled ones
    assert lib.dbst_block_sparse_attn_raster(a, a, a, ctypes.byref(g), None, a, None, 0.0, a, None,
                                             None) == dbst.DBST_EINVAL
    assert lib.dbst_block_sparse_attn_raster(a, ctypes.c_void_p((1 << 20) + 8), a, ctypes.byref(g), a, a, None, 0.0, a,
                                             None, None) == dbst.DBST_EINVAL
    assert lib.dbst_block_sparse_attn_raster(a, a, a, ctypes.byref(g), a, a, ctypes.c_void_p((1 << 20) + 2), 0.0, a,
                                             None, None) == dbst.DBST_EINVAL   # misaligned pair list
    assert lib.dbst_pair_query_blocks(None, ctypes.byref(g), a, None) == dbst.DBST_EINVAL
    assert lib.dbst_pair_query_blocks(a, ctypes.byref(g), ctypes.c_void_p((1 << 20) + 1), None) == dbst.DBST_EINVAL
    assert lib.dbst_pair_query_blocks(a, None, a, None) == dbst.DBST_EINVAL
    assert lib.dbst_dense_attn_raster(a, a, a, ctypes.byref(g), float("inf"), a, None, None) == dbst.DBST_EINVAL
    assert lib.dbst_dense_attn_raster(None, a, a, ctypes.byref(g), 0.0, a, None, None) == dbst.DBST_EINVAL
    ws = lib.dbst_mask_workspace_bytes(ctypes.byref(g))
    assert lib.dbst_build_block_mask_raster(None, a, ctypes.byref(g), 0.9, -1, a, a, a, a, ws, None) == dbst.DBST_EINVAL
    assert lib.dbst_build_block_mask_raster(a, a, ctypes.byref(g), 0.9, -1, a, a, a, a, ws - 1, None) == dbst.DBST_EINVAL
    assert lib.dbst_build_block_mask_raster(a, a, ctypes.byref(g), 1.5, -1, a, a, a, a, ws, None) == dbst.DBST_EINVAL


@pytest.mark.parametrize("p", [0.0, -0.5, 1.0000001, 2.0, float("nan")])
def test_build_mask_rejects_p_outside_unit_interval(lib, p):
    g = geom()
    a = ctypes.c_void_p(1 << 20)
    ws = lib.dbst_mask_workspace_bytes(ctypes.byref(g))
    assert lib.dbst_build_block_mask(a, a, ctypes.byref(g), p, -1, a, a, a, a, ws, None) == dbst.DBST_EINVAL


def test_build_mask_rejects_small_workspace(lib):
    g = geom()
    a = ctypes.c_void_p(1 << 20)
    ws = lib.dbst_mask_workspace_bytes(ctypes.byref(g))
    assert lib.dbst_build_block_mask(a, a, ctypes.byref(g), 0.9, -1, a, a, a, a, ws - 1, None) == dbst.DBST_EINVAL


def test_workspace_size_formula(lib):
    g = geom(B=2, H=3, D=64, grid=(8, 16, 16), tile=(1, 8, 8))
    nb, bh = 32, 6

    def up(x):
        return (x + 255) // 256 * 256
    # float64 layout (SIP mask, rows of more than 2048 blocks): block means of q and k, pooled logits
    f64 = 2 * up(bh * nb * 64 * 8) + up(bh * nb * nb * 8)
    # tensor-core layout: per-head max key norm and the refine-list length, 6 bf16 pieces and 2 float32
    # residuals of the means, 2 norms per block, the float32 pooled logits, the refine list
    tc = (up((bh + 1) * 4) + up(6 * bh * nb * 64 * 2) + up(2 * bh * nb * 64 * 4) + up(2 * bh * nb * 4) +
          up(bh * nb * nb * 4) + up(bh * nb * 8))
    assert lib.dbst_mask_workspace_bytes(ctypes.byref(g)) == max(f64, tc)


def test_python_binding_validates_shapes_before_calling():
    import torch
    g = geom()
    x = torch.zeros((1, 2, g.N, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dbst.tile_reorder(x, g)          # not a CUDA tensor


def test_backward_entry_points_validate_arguments(lib):
    g = geom()
    a = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    ws = lib.dbst_attn_backward_workspace_bytes(ctypes.byref(g))
    assert ws == (1 * 2 * g.N * 8 + 255) // 256 * 256
    assert lib.dbst_attn_backward_workspace_bytes(ctypes.byref(geom(D=96))) == 0
    for fn in (lib.dbst_block_sparse_attn_backward, lib.dbst_block_sparse_attn_backward_raster):
        ok = [a, a, a, a, a, ctypes.byref(g), a, a, a, a, 0.0, a, a, a, a, ws, None]
        for i in (0, 1, 2, 3, 4, 6, 7, 8, 9, 11, 12, 13, 14):          # each pointer null
            args = list(ok)
            args[i] = None
            assert fn(*args) == dbst.DBST_EINVAL, i
        for i in (0, 4, 7, 9, 11, 14):                                 # misaligned
            args = list(ok)
            args[i] = odd
            assert fn(*args) == dbst.DBST_EINVAL, i
        args = list(ok)
        args[3] = ctypes.c_void_p((1 << 20) + 2)                       # lse not 4-byte aligned
        assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[15] = ws - 1                                              # workspace too small
        assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[10] = float("nan")
        assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[5] = ctypes.byref(geom(D=96))
        assert fn(*args) == dbst.DBST_EINVAL
    assert lib.dbst_transpose_block_mask(a, ctypes.byref(g), a, a, a, None) == dbst.DBST_EINVAL   # in place
    assert lib.dbst_transpose_block_mask(None, ctypes.byref(g), a, a, a, None) == dbst.DBST_EINVAL
    assert lib.dbst_transpose_block_mask(a, ctypes.byref(g), ctypes.c_void_p(1 << 30), odd, a, None) == dbst.DBST_EINVAL
    assert lib.dbst_transpose_block_mask(a, None, ctypes.c_void_p(1 << 30), a, a, None) == dbst.DBST_EINVAL


def test_squad_entry_point_validates_shapes(lib):
    a = ctypes.c_void_p(1 << 20)
    tb = 2 * 16384 * 128 * 2
    assert lib.dbst_squad_workspace_bytes(1, 2, 16384, 128, 128) == 4 * tb
    for B, H, N, D, w in ((1, 2, 16384, 96, 128), (1, 2, 16384, 128, 100), (1, 2, 16384, 128, 32),
                          (1, 2, 8192, 128, 256), (0, 2, 16384, 128, 128), (1, 2, 16000, 128, 128)):
        assert lib.dbst_squad_workspace_bytes(B, H, N, D, w) == 0, (N, D, w)   # N/w=32 is rejected too
        assert lib.dbst_squad_attn(a, a, a, B, H, N, D, w, 0.0, a, a, 1 << 40, None) == dbst.DBST_EINVAL
    ok = (1, 2, 16384, 128, 128)
    assert lib.dbst_squad_attn(a, a, a, *ok, 0.0, a, a, 4 * tb - 1, None) == dbst.DBST_EINVAL
    assert lib.dbst_squad_attn(None, a, a, *ok, 0.0, a, a, 4 * tb, None) == dbst.DBST_EINVAL
    assert lib.dbst_squad_attn(a, a, ctypes.c_void_p((1 << 20) + 8), *ok, 0.0, a, a, 4 * tb, None) == dbst.DBST_EINVAL
    assert lib.dbst_squad_attn(a, a, a, *ok, float("nan"), a, a, 4 * tb, None) == dbst.DBST_EINVAL


def test_sip_and_offset_entry_points_validate_arguments(lib):
    g = geom()
    a = ctypes.c_void_p(1 << 20)
    odd = ctypes.c_void_p((1 << 20) + 8)
    ws = lib.dbst_mask_workspace_bytes(ctypes.byref(g))
    for fn in (lib.dbst_build_sip_mask, lib.dbst_build_sip_mask_raster):
        ok = [a, a, ctypes.byref(g), 4.0, a, a, a, a, a, a, ws, None]
        for i in (0, 1, 4, 5, 6, 7, 8, 9):
            args = list(ok)
            args[i] = None
            assert fn(*args) == dbst.DBST_EINVAL, i
            args[i] = odd
            assert fn(*args) == dbst.DBST_EINVAL, i
        for budget in (0.0, -1.0, float("nan"), float("inf")):
            args = list(ok)
            args[3] = budget
            assert fn(*args) == dbst.DBST_EINVAL, budget
        args = list(ok)
        args[10] = ws - 1
        assert fn(*args) == dbst.DBST_EINVAL
    for fn in (lib.dbst_block_sparse_attn_offsets, lib.dbst_block_sparse_attn_offsets_raster):
        ok = [a, a, a, ctypes.byref(g), a, a, None, 0.0, a, None, None]
        for i in (0, 1, 2, 4, 5, 8):
            args = list(ok)
            args[i] = None
            assert fn(*args) == dbst.DBST_EINVAL, i
        args = list(ok)
        args[6] = ctypes.c_void_p((1 << 20) + 2)                       # offsets not 4-byte aligned
        assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[7] = float("nan")
        assert fn(*args) == dbst.DBST_EINVAL


def test_mask_builders_reject_too_many_heads_before_any_launch(lib):
    """B*H above the pooled-logits grid limit is refused before anything is enqueued (the
    refusal must not depend on a launch failing)."""
    g = geom(B=1, H=70000, D=64, grid=(1, 8, 8), tile=(1, 8, 8))
    a = ctypes.c_void_p(1 << 20)
    ws = lib.dbst_mask_workspace_bytes(ctypes.byref(g))
    assert ws > 0
    assert lib.dbst_build_block_mask(a, a, ctypes.byref(g), 0.9, -1, a, a, a, a, ws, None) == dbst.DBST_EINVAL
    assert lib.dbst_build_block_mask_raster(a, a, ctypes.byref(g), 0.9, -1, a, a, a, a, ws, None) == dbst.DBST_EINVAL
    assert lib.dbst_build_sip_mask(a, a, ctypes.byref(g), 2.0, a, a, a, a, a, a, ws, None) == dbst.DBST_EINVAL


def test_fine_mask_and_group_attention_validate_arguments(lib):
    g = geom()
    a = ctypes.c_void_p(1 << 20)
    ws = lib.dbst_fine_mask_workspace_bytes(ctypes.byref(g))
    nb, ng, bh = g.N // 64, g.N // 4, 2
    up = lambda x: (x + 255) // 256 * 256   # noqa: E731
    assert ws == up(bh * nb * 128 * 8) + up(bh * ng * 128 * 8) + up(bh * nb * ng * 8)
    big = geom(grid=(8, 128, 128), tile=(1, 8, 8))          # 2048 blocks: above the 1024 limit
    assert lib.dbst_fine_mask_workspace_bytes(ctypes.byref(big)) == 0
    for fn in (lib.dbst_build_fine_mask, lib.dbst_build_fine_mask_raster):
        ok = [a, a, ctypes.byref(g), 0.9, a, a, a, a, ws, None]
        for i in (0, 1, 4, 5, 6, 7):
            args = list(ok)
            args[i] = None
            assert fn(*args) == dbst.DBST_EINVAL, i
        for p in (0.0, 1.5, float("nan")):
            args = list(ok)
            args[3] = p
            assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[8] = ws - 1
        assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[2] = ctypes.byref(big)
        assert fn(*args) == dbst.DBST_EINVAL
    for fn in (lib.dbst_block_sparse_attn_groups, lib.dbst_block_sparse_attn_groups_raster):
        ok = [a, a, a, ctypes.byref(g), a, a, a, 0.0, a, None, None]
        for i in (0, 1, 2, 4, 5, 6, 8):
            args = list(ok)
            args[i] = None
            assert fn(*args) == dbst.DBST_EINVAL, i
        args = list(ok)
        args[6] = ctypes.c_void_p((1 << 20) + 1)                      # group mask not 2-byte aligned
        assert fn(*args) == dbst.DBST_EINVAL


def test_gathered_group_attention_validates_arguments(lib):
    g = geom()
    a = ctypes.c_void_p(1 << 20)
    for fn in (lib.dbst_block_sparse_attn_gather, lib.dbst_block_sparse_attn_gather_raster):
        ok = [a, a, a, ctypes.byref(g), a, 0.0, a, None, None]
        for i in (0, 1, 2, 4, 6):
            args = list(ok)
            args[i] = None
            assert fn(*args) == dbst.DBST_EINVAL, i
        args = list(ok)
        args[4] = ctypes.c_void_p((1 << 20) + 1)
        assert fn(*args) == dbst.DBST_EINVAL
        args = list(ok)
        args[3] = ctypes.byref(geom(grid=(8, 128, 128), tile=(1, 8, 8)))   # 2048 blocks
        assert fn(*args) == dbst.DBST_EINVAL
    narrow = geom(grid=(4, 16, 16), tile=(4, 8, 2))                       # tx = 2: no 4-token run along x
    assert lib.dbst_block_sparse_attn_gather_raster(a, a, a, ctypes.byref(narrow), a, 0.0, a, None,
                                                    None) == dbst.DBST_EINVAL
