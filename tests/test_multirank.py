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
