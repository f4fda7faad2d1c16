"""The bench's multi-rank logic on two CPU ranks (gloo): every rank times its own
independent problem, the job time is the max over ranks, and the job throughput
counts every rank's work (weak scaling)."""
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r was slower in one measurement and faster in another
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 5.0], world, "cpu")
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        assert out[0] == out[1] == [2.0, 10.0, 5.0]


def test_job_throughput_counts_every_rank():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.job_tflops(1, 3.0e12, 10.0)
    assert one == pytest.approx(300.0)
    assert bench.job_tflops(4, 3.0e12, 10.0) == pytest.approx(4 * one)


def test_reference_arm_non_zero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--steps", "1", "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0
    assert r.stdout.strip() == ""


def test_reference_arm_rank_zero_prints_the_contract_line():
    """The oracle arm on rank 0: one JSON line with the metric, a positive value, the oracle as its own
    cpu_baseline and an end-to-end figure equal to the value with no host copies."""
    import json
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--ref-budget", "0.5"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


# ---------------------------------------------------------------- head split (shard.py)
def _oracle_local(q, k, v, gl, p, sta):
    """The oracle on one rank's heads, in place of the CUDA path: raster bf16 q, k, v -> raster (o, lse), float64."""
    import numpy as np
    import torch
    import oracle as O
    og = O.Geometry(gl.B, gl.H, gl.D, gl.T, gl.Y, gl.X, gl.tt, gl.ty, gl.tx)
    qt, kt, vt = (O.tile_reorder(t.view(torch.int16).numpy().view(np.uint16), og) for t in (q, k, v))
    mask = O.build_block_mask(qt, kt, og, p, sta)
    o, lse = O.masked_attention(qt, kt, vt, mask, 64, 1.0 / np.sqrt(gl.D))
    return (torch.from_numpy(O.tile_unreorder(o, og)),
            torch.from_numpy(O.tile_unreorder(lse[..., None], og)[..., 0]))


def _split_workload(H):
    import dbst_synth as S
    return S.Workload("split", 1, B=2, H=H, D=64, grid=(4, 8, 8), tile=(1, 8, 8), alpha=0.7, beta=0.3, f_rms=2.0,
                      kmax=3, p_list=(0.9,), sta_radius=-1)


def _shard_main(rank, world, port, out, H, p):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import dbst_synth as S
    from dynamic_block_sparse_tile_b200 import Geom, shard
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = _split_workload(H)
        g = Geom.make(w.B, w.H, w.D, w.grid, w.tile)
        tq, tk, tv = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) for a in S.make_qkv(w))
        o, lse = shard.run_sharded(tq, tk, tv, g, p, world, rank, local_fn=_oracle_local)
        out[rank] = (o.numpy(), lse.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_head_range_partitions_the_heads():
    sys.path.insert(0, ROOT)
    from dynamic_block_sparse_tile_b200 import shard
    for H in (1, 2, 3, 8, 24, 40):
        for world in (1, 2, 3, 4, 8):
            ranges = [shard.head_range(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and sizes == sorted(sizes, reverse=True)
    with pytest.raises(ValueError):
        shard.head_range(8, 2, 2)


@pytest.mark.parametrize("H", [4, 3])
def test_head_split_on_two_gloo_ranks_equals_the_whole_job(H):
    """Two CPU ranks each run their heads (the oracle standing in for the CUDA path) with no collective, then
    gather o and lse: every rank must hold exactly the single-process result for all heads."""
    import numpy as np
    import torch
    sys.path.insert(0, ROOT)
    import dbst_synth as S
    from dynamic_block_sparse_tile_b200 import Geom
    p = 0.9
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_shard_main, args=(world, port, out, H, p), nprocs=world, join=True)
        got = [out[r] for r in range(world)]
    w = _split_workload(H)
    g = Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    tq, tk, tv = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) for a in S.make_qkv(w))
    o_ref, lse_ref = _oracle_local(tq, tk, tv, g, p, -1)
    for o, lse in got:
        np.testing.assert_array_equal(o, o_ref.numpy())
        np.testing.assert_array_equal(lse, lse_ref.numpy())
