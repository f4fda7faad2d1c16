"""The allocation-free mask entry point (dbst_build_block_mask_noalloc).

Some callers cannot allocate device memory while they run — a serving loop or
plugin host that owns every byte of device memory and forbids cudaMalloc
after start-up has no workspace to lend.  The allocation-free entry point
serves them from a fixed static scratch array inside the library.  This test
calls it through the C ABI and checks that it reproduces the regular entry
point's output exactly, on two calls in a row (the second call reuses the
scratch the first one left behind), and that a shape too large for the
static scratch is refused before anything runs.

Kept in a file of its own that sorts last among the core path's tests, so that
a run which stops at the first failure has already run every other core test
(tests/conftest.py runs the extension rows' tests after it).
"""
import ctypes

import numpy as np
import pytest
import torch

import dbst_synth as S
import oracle as O
import dynamic_block_sparse_tile_b200 as dbst
from dynamic_block_sparse_tile_b200 import build as dbst_build
from tests import parity as P

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    dbst_build.build()
    return dbst.load()


def tiled_inputs(w, heads=None):
    q, k, _ = S.make_qkv(w, heads=heads)
    g = P.geometry(w, q.shape[1])
    return P.bits_to_torch(O.tile_reorder(q, g)), P.bits_to_torch(O.tile_reorder(k, g))


@pytest.mark.parametrize("name,p,sta,heads", [("small", 0.9, 1, None), ("sweep", 0.8, -1, None),
                                              ("tiny", 0.9, -1, None)])
def test_noalloc_matches_regular_entry_point_twice(lib, name, p, sta, heads):
    w = S.workload(name)
    qt, kt = tiled_inputs(w, heads)
    g = dbst.Geom.make(w.B, qt.shape[1], w.D, w.grid, w.tile)
    ref = dbst.build_block_mask(qt, kt, g, p, sta)
    dbst.get_error()
    ref = [t.cpu().numpy() for t in ref]
    for call in range(2):
        out = (torch.full_like(torch.from_numpy(ref[0]), -1).cuda(), torch.full_like(torch.from_numpy(ref[1]), -1).cuda(),
               torch.full_like(torch.from_numpy(ref[2]), -1).cuda())
        torch.cuda.synchronize()
        before = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
        status = lib.dbst_build_block_mask_noalloc(
            ctypes.c_void_p(qt.data_ptr()), ctypes.c_void_p(kt.data_ptr()), ctypes.byref(g), ctypes.c_float(p),
            ctypes.c_int(sta), ctypes.c_void_p(out[0].data_ptr()), ctypes.c_void_p(out[1].data_ptr()),
            ctypes.c_void_p(out[2].data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert status == dbst.DBST_OK, status
        dbst.get_error()
        # nothing was allocated: the device's free memory (cudaMemGetInfo) and torch's pools are as before
        after = (torch.cuda.mem_get_info()[0], torch.cuda.memory_allocated(), torch.cuda.memory_reserved())
        assert after == before, f"call {call}: device memory changed from {before} to {after}"
        bits, cnt, idx = (t.cpu().numpy() for t in out)
        np.testing.assert_array_equal(bits, ref[0], err_msg=f"call {call}: mask bits")
        np.testing.assert_array_equal(cnt, ref[1], err_msg=f"call {call}: kv_count")
        for pos in np.ndindex(*cnt.shape):
            n = cnt[pos]
            np.testing.assert_array_equal(idx[pos][:n], ref[2][pos][:n], err_msg=f"call {call}: kv_idx {pos}")


def test_noalloc_refuses_shapes_beyond_the_static_scratch(lib):
    w = S.workload("wan")
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    assert dbst.mask_workspace_bytes(g) > dbst.NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(1 << 20)
    status = lib.dbst_build_block_mask_noalloc(a, a, ctypes.byref(g), ctypes.c_float(0.9), ctypes.c_int(-1),
                                               a, a, a, None)
    assert status == dbst.DBST_ETOOLARGE
    with pytest.raises(dbst.DbstError) as e:
        x = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.bfloat16, device="cuda")
        dbst.build_block_mask_noalloc(x, x, g, 0.9)
    assert e.value.status == dbst.DBST_ETOOLARGE
