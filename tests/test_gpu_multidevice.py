"""One process driving two GPUs: the head split of shard.py with rank = device.

The library keeps per-device state (the opt-in to large dynamic shared
memory, the multiprocessor count, the static scratch's address), so one
process may call it on several devices.  Each device runs the fused path on
its heads; the concatenated results must equal a single-device run over all
heads bit for bit, since every head is computed on its own.  Skipped on a
machine with fewer than two GPUs.
"""
import numpy as np
import pytest
import torch

import dbst_synth as S
import dynamic_block_sparse_tile_b200 as dbst
from dynamic_block_sparse_tile_b200 import shard

pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available() or torch.cuda.device_count() < 2,
                                 reason="needs two GPUs")]


@pytest.mark.parametrize("name,p,sta", [("small", 0.9, 1), ("sweep", 0.7, -1)])
def test_two_devices_in_one_process_match_one_device(name, p, sta):
    from dynamic_block_sparse_tile_b200 import build
    build.build()
    w = S.workload(name)
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    host = [torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) for a in S.make_qkv(w)]
    with torch.cuda.device(0):
        o_full, lse_full = shard.run_local(*(t.cuda() for t in host), g, p, sta)
        o_full, lse_full = o_full.cpu(), lse_full.cpu()
    parts = []
    for dev in (0, 1):
        h0, h1 = shard.head_range(w.H, 2, dev)
        with torch.cuda.device(dev):
            qkv = [shard.local_heads(t, h0, h1).to(f"cuda:{dev}") for t in host]
            o, lse = shard.run_local(*qkv, shard.head_geometry(g, h0, h1), p, sta)
            parts.append((o.cpu(), lse.cpu()))
    o = torch.cat([a for a, _ in parts], dim=1)
    lse = torch.cat([b for _, b in parts], dim=1)
    assert torch.equal(o.view(torch.int16), o_full.view(torch.int16))
    assert torch.equal(lse, lse_full)
