"""Benchmark of the block-sparse tile attention path on B200.

One step = one pass of the whole path over one batch of the Wan-like 480p
latent workload (B=1, H=40, D=128, token grid 21x32x56 in 1x8x8 tiles,
N=37632, 588 blocks; CDF threshold p=0.9; seeded synthetic q/k/v).  Default
(`--path fused`): raster q, k, v in, raster o out, the tile reorder done by the
kernels' own loads and stores:
    build_block_mask_raster(q, k) -> pair_query_blocks -> block_sparse_attn_raster(q, k, v, pairs) -> o
(8 launches: a memset and five kernels for the mask (block means, pooled logits on the tensor cores,
row selection, float64 refinement of the rows whose error band holds several blocks, and of the
rare rows whose band is wider than a warp), the query-block pairing, the attention).  `--path
explicit` runs the same steps as separate passes (11 launches, no pairing):
    tile_reorder(q, k, v) -> build_block_mask -> block_sparse_attn -> tile_unreorder(o)

`value` = kept-block TFLOP/s of the whole step (4*D*64*64 FLOP per kept
block pair, summed over heads, divided by the step time) with inputs resident
in HBM; `e2e` = the same metric with pinned-host inputs copied in and the
output copied back inside the timed region.  Inputs (385 MB per tensor) are
larger than the 126 MB L2, so no flush is needed between steps.

Multi-GPU (torchrun): every rank runs its own independent Wan-sized problem
(weak scaling, no collective on the data path); the time is the max over
ranks.  `--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import dbst_synth as S  # noqa: E402

METRIC = "sparse-attn ms/call & TFLOP/s on kept blocks (N=32760,H=40,D=128,bf16)"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], d["bf16_tflops"], d["bf16_tflops_sustained"], "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def source_digest(texts) -> str:
    """sha256 (first 16 hex digits) of C++ sources with // comments and blank space removed, so a
    measurement stays attached to its code across edits that touch only comments."""
    import hashlib
    import re
    h = hashlib.sha256()
    for text in texts:
        code = "\n".join(" ".join(re.sub(r"//.*", "", line).split()) for line in text.splitlines())
        h.update(re.sub(r"\n+", "\n", code).strip().encode())
    return h.hexdigest()[:16]


def attn_source_digest() -> str:
    texts = []
    for f in ("attn_pair.cuh", "ptx.cuh"):
        with open(os.path.join(ROOT, "dynamic_block_sparse_tile_b200", "csrc", f)) as fh:
            texts.append(fh.read())
    return source_digest(texts)


def measured_traffic(workload: str, p: float, layout: str):
    """DRAM bytes per attention launch from the committed ncu summary, if it matches this kernel source."""
    path = os.path.join(ROOT, "profiles", "pair_attn_kernel_dram_traffic.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    for line in text.splitlines():
        if line.startswith("| ") and f"`{workload}`" in line and f"p={p}" in line and layout in line:
            cells = [c.strip() for c in line.strip("|").split("|")]
            try:
                digest, total = cells[1].strip("`"), float(cells[4])
            except (IndexError, ValueError):
                continue
            if digest == attn_source_digest():
                return total
    return None


def workload_desc(w: S.Workload, p: float) -> str:
    return (f"{w.name}-like latent: B={w.B} H={w.H} D={w.D} grid={w.grid[0]}x{w.grid[1]}x{w.grid[2]} "
            f"(N={w.N}, {w.NB} blocks of {w.tile[0]}x{w.tile[1]}x{w.tile[2]}), p={p}, "
            f"sta_radius={w.sta_radius}")


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_model() -> str:
    """The host CPU's model name, from /proc/cpuinfo where it exists."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# NVIDIA's dense bf16 tensor figure for one B200 (its 4.5 PFLOP/s per-GPU figure assumes 2:4
# sparsity); reported beside the measured peaks, never instead of them.
NOMINAL_BF16_TFLOPS = 2250.0


def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def oracle_sample(w: S.Workload, p: float, budget_s: float, seed: int = 7):
    """Time the CPU oracle on a bounded sample of the workload.

    Sample: a few heads; for each, the full oracle mask (pool, reduced map,
    CDF selection) and the masked attention of randomly chosen query blocks,
    until ~budget_s seconds of CPU work.  Returns (kept-block TFLOP/s, seconds,
    description).
    """
    import dataclasses
    import oracle as O
    rng = np.random.default_rng(seed)
    g1 = O.Geometry(1, 1, w.D, *w.grid, *w.tile)
    scale = 1.0 / math.sqrt(w.D)
    flops = 0.0
    elapsed = 0.0
    heads_done, rows_done = 0, 0
    h = 0
    while elapsed < budget_s and h < w.H:
        q, k, v = S.make_qkv(w, heads=range(h, h + 1), batches=range(1))
        t0 = time.perf_counter()
        qt, kt, vt = (O.tile_reorder(a, g1) for a in (q, k, v))
        mask = O.build_block_mask(qt, kt, g1, p, w.sta_radius)
        elapsed += time.perf_counter() - t0
        heads_done += 1
        order = rng.permutation(g1.NB)
        for i in order:
            if elapsed >= budget_s:
                break
            t0 = time.perf_counter()
            O.masked_attention(qt, kt, vt, mask, 64, scale, rows=[(0, 0, int(i))])
            elapsed += time.perf_counter() - t0
            flops += 4.0 * w.D * 64 * 64 * float(mask[0, 0, i].sum())
            rows_done += 1
        h += 1
    desc = (f"oracle (numpy fp64) on {heads_done} head(s): full mask build per head + masked attention of "
            f"{rows_done} random query blocks; kept-block FLOPs of those blocks / CPU seconds")
    return flops / elapsed / 1e12, elapsed, desc


def max_over_ranks(vals, world: int, device: str):
    """Element-wise max over ranks of per-rank timings: the slowest rank sets the job's time."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(vals), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.tolist()]


def job_tflops(world: int, flops_per_rank: float, ms_per_step: float) -> float:
    """Whole-job throughput under weak scaling: every rank runs its own problem of flops_per_rank per step."""
    return world * flops_per_rank / (ms_per_step * 1e-3) / 1e12


def run_reference(args, w, p):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals, secs = [], []
    desc = ""
    # bounded: about two minutes of oracle work for the whole run, however many steps
    budget = args.ref_budget if args.ref_budget > 0 else max(2.0, 120.0 / (args.warmup + args.steps))
    for step in range(args.warmup + args.steps):
        v, s, desc = oracle_sample(w, p, budget_s=budget, seed=100 + step)
        if step >= args.warmup:
            vals.append(v)
            secs.append(s)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * statistics.mean(secs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": workload_desc(w, p), "sample": "bounded oracle sample"},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                             "sample": desc, "cpu_model": cpu_model(), "nproc": os.cpu_count()},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def timed_median(fn, steps: int, warmup: int) -> float:
    """Median CUDA-event time (ms) of fn() on the current stream over `steps` calls, after
    max(warmup, 3) untimed calls."""
    import torch
    for _ in range(max(warmup, 3)):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(steps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def run_sweep(args, w):
    print(json.dumps(measure_sweep(args, w)), flush=True)
    return 0


def measure_sweep(args, w) -> dict:
    """Attention time and kept-block TFLOP/s against the kept fraction; dense attention at the same shape."""
    import torch
    import dynamic_block_sparse_tile_b200 as dbst
    dbst.load()
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in S.make_qkv(w))
    qt, kt, vt = (dbst.tile_reorder(x, g) for x in (q, k, v))
    ot = torch.empty_like(qt)
    lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device="cuda")

    def timed(fn, reps):
        return timed_median(fn, reps, 3)

    dense_ms = timed(lambda: dbst.dense_attn(qt, kt, vt, g), args.steps)
    dense_flops = 4.0 * w.D * w.N * w.N * w.B * w.H
    _, bf16, _, src = peaks()
    rows = []
    for p in w.p_list:
        bits, cnt, idx = dbst.build_block_mask(qt, kt, g, p, w.sta_radius)
        mask_ms = timed(lambda: dbst.build_block_mask(qt, kt, g, p, w.sta_radius), args.steps)
        ms = timed(lambda: dbst.block_sparse_attn(qt, kt, vt, g, cnt, idx, 0.0, True, ot, lse), args.steps)
        kept = int(cnt.sum().item())
        fl = 4.0 * w.D * 64 * 64 * kept
        rows.append({"p": p, "kept_fraction": kept / (g.B * g.H * g.NB * g.NB), "sparse_attn_ms": ms,
                     "kept_tflops": fl / (ms * 1e-3) / 1e12, "frac_of_bf16_peak": fl / (ms * 1e-3) / 1e12 / bf16,
                     "mask_build_ms": mask_ms, "speedup_vs_dense": dense_ms / ms})
    # dense again at the end: the GPU runs under its power cap, so the first and last points
    # of a sweep can see different clocks; the crossover uses the slower of the two dense times
    dense_end_ms = timed(lambda: dbst.dense_attn(qt, kt, vt, g), args.steps)
    dbst.get_error()
    dense_ref = max(dense_ms, dense_end_ms)
    for r in rows:
        r["speedup_vs_dense"] = dense_ref / r["sparse_attn_ms"]
    crossover = next((r["kept_fraction"] for r in rows if r["sparse_attn_ms"] >= dense_ref), None)
    return {"sweep": workload_desc(w, float("nan")), "dense_attn_ms": dense_ms, "dense_attn_ms_end": dense_end_ms,
            "dense_tflops": dense_flops / (dense_ms * 1e-3) / 1e12, "peak_source": src, "points": rows,
            "dense_crossover_kept_fraction": crossover,
            "crossover_note": "kept fraction of the first p whose sparse attention is no faster than dense; "
                              "null: sparse is faster at every p of the sweep, p = 1 (every block kept) included"}


def measure_backward(args, w, p, qkv=None) -> dict:
    """Backward of the block-sparse attention (raster layout) on one GPU: mask, its transpose, forward
    for the log-sum-exp, then the timed backward."""
    import torch
    import dynamic_block_sparse_tile_b200 as dbst
    dbst.load()
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()   # noqa: E731
    q, k, v = qkv if qkv is not None else (to_dev(a) for a in S.make_qkv(w))
    do = to_dev(S.make_grad(w))
    bits, cnt, idx = dbst.build_block_mask_raster(q, k, g, p, w.sta_radius)
    pairs = dbst.pair_query_blocks(bits, g)
    o, lse = dbst.block_sparse_attn_raster(q, k, v, g, cnt, idx, pairs=pairs)
    out_t = dbst.transpose_block_mask(bits, g)
    _, qcnt, qidx = out_t
    ws = torch.empty(dbst.attn_backward_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    grads = tuple(torch.empty_like(q) for _ in range(3))
    fwd_ms = timed_median(lambda: dbst.block_sparse_attn_raster(q, k, v, g, cnt, idx, 0.0, True, o, lse, pairs),
                          args.steps, args.warmup)
    tr_ms = timed_median(lambda: dbst.transpose_block_mask(bits, g, out=out_t), args.steps, args.warmup)
    bwd_ms = timed_median(lambda: dbst.block_sparse_attn_backward(q, k, v, lse, do, g, cnt, idx, qcnt, qidx,
                                                                  raster=True, workspace=ws, out=grads),
                          args.steps, args.warmup)
    dbst.get_error()
    kept = int(cnt.sum().item())
    unit = 2.0 * w.D * 64 * 64 * kept            # one 64x64xD product over every kept block pair
    _, bf16, _, src = peaks()
    return {"backward": workload_desc(w, p), "kept_fraction": kept / (g.B * g.H * g.NB * g.NB),
            "backward_ms": bwd_ms, "forward_attn_ms": fwd_ms, "transpose_ms": tr_ms,
            "backward_tflops": 5 * unit / (bwd_ms * 1e-3) / 1e12,
            "backward_tensor_tflops": 9 * unit / (bwd_ms * 1e-3) / 1e12,
            "forward_tflops": 2 * unit / (fwd_ms * 1e-3) / 1e12,
            "bf16_peak_tflops": bf16, "peak_source": src,
            "note": "backward_tflops counts the 5 products of the gradient (S, dP, dV, dK, dQ); the kernels "
                    "run 9 (S and dP twice more: the delta sweep of the dq pass and the dk/dv pass)"}


def run_backward(args, w, p):
    print(json.dumps(measure_backward(args, w, p)), flush=True)
    return 0


def measure_sip(args, w, p, qkv=None) -> dict:
    """SIP on one workload: sampled mask with inclusion-probability offsets at the NABLA mask's mean
    kept count per row, then the offset attention; plus that attention without offsets on the
    NABLA mask."""
    import torch
    import dynamic_block_sparse_tile_b200 as dbst
    dbst.load()
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()   # noqa: E731
    q, k, v = qkv if qkv is not None else (to_dev(a) for a in S.make_qkv(w))
    bits, cnt, idx = dbst.build_block_mask_raster(q, k, g, p, w.sta_radius)
    budget = float(cnt.double().mean().item())
    gen = torch.Generator(device="cuda").manual_seed(1234)
    u = torch.rand((g.B, g.H, g.NB, g.NB), dtype=torch.float64, device="cuda", generator=gen)
    ws = torch.empty(dbst.mask_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    sip = dbst.build_sip_mask(q, k, g, budget, u, raster=True, workspace=ws)
    o = torch.empty_like(q)
    lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device="cuda")
    sel_ms = timed_median(lambda: dbst.build_sip_mask(q, k, g, budget, u, raster=True, workspace=ws, out=sip),
                          args.steps, args.warmup)
    sip_pairs = dbst.pair_query_blocks(sip[0], g)
    attn_ms = timed_median(lambda: dbst.block_sparse_attn_offsets(q, k, v, g, sip[1], sip[2], sip[3], raster=True,
                                                                  out=o, lse=lse, pairs=sip_pairs),
                           args.steps, args.warmup)
    plain_ms = timed_median(lambda: dbst.block_sparse_attn_offsets(q, k, v, g, cnt, idx, None, raster=True, out=o,
                                                                   lse=lse), args.steps, args.warmup)
    pairs = dbst.pair_query_blocks(bits, g)
    fwd_ms = timed_median(lambda: dbst.block_sparse_attn_raster(q, k, v, g, cnt, idx, 0.0, True, o, lse, pairs),
                          args.steps, args.warmup)
    dbst.get_error()
    kept_sip = int(sip[1].sum().item())
    kept = int(cnt.sum().item())
    unit = 4.0 * w.D * 64 * 64
    return {"sip": workload_desc(w, p), "budget_blocks_per_row": budget,
            "kept_fraction_sip": kept_sip / (g.B * g.H * g.NB * g.NB), "sip_mask_ms": sel_ms,
            "sip_attn_ms": attn_ms, "sip_attn_tflops": unit * kept_sip / (attn_ms * 1e-3) / 1e12,
            "offset_attn_on_nabla_mask_ms": plain_ms,
            "offset_attn_on_nabla_mask_tflops": unit * kept / (plain_ms * 1e-3) / 1e12,
            "forward_on_nabla_mask_ms": fwd_ms,
            "sip_attn_over_forward": attn_ms / fwd_ms,
            "note": "TFLOP/s count the 2 products of attention per kept block pair; the offsets ride in the "
                    "forward kernel's exponent; SIP attention and the forward run on the pair lists of "
                    "dbst_pair_query_blocks for their masks, the offset kernel on the NABLA mask without one"}


def run_sip(args, w, p):
    print(json.dumps(measure_sip(args, w, p)), flush=True)
    return 0


def measure_step(args, name: str) -> dict:
    """The fused step (mask build + pairing + attention, raster in and out) on another workload,
    timed call by call: the Wan-like latent in its 2x4x8 tiles."""
    import torch
    import dynamic_block_sparse_tile_b200 as dbst
    dbst.load()
    w = S.workload(name)
    p = w.p_list[0]
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in S.make_qkv(w))
    ws = torch.empty(dbst.mask_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    mask = dbst.build_block_mask_raster(q, k, g, p, w.sta_radius, workspace=ws)
    pairs = dbst.pair_query_blocks(mask[0], g)
    o = torch.empty_like(q)
    lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device="cuda")

    mask_ms = timed_median(lambda: dbst.build_block_mask_raster(q, k, g, p, w.sta_radius, workspace=ws, out=mask),
                           args.steps, args.warmup)
    pairing_ms = timed_median(lambda: dbst.pair_query_blocks(mask[0], g, out=pairs), args.steps, args.warmup)
    attn_ms = timed_median(lambda: dbst.block_sparse_attn_raster(q, k, v, g, mask[1], mask[2], 0.0, True, o, lse,
                                                                 pairs), args.steps, args.warmup)
    dbst.get_error()
    kept = int(mask[1].sum().item())
    flops = 4.0 * w.D * 64 * 64 * kept
    hbm, bf16, _, src = peaks()
    mask_gbs = 2 * w.B * w.H * w.N * w.D * 2 / (mask_ms * 1e-3) / 1e9
    return {"workload": workload_desc(w, p), "kept_fraction": kept / (g.B * g.H * g.NB * g.NB),
            "mask_build_ms": mask_ms, "mask_build_gbs": mask_gbs, "mask_frac_of_hbm": mask_gbs / hbm,
            "pairing_ms": pairing_ms, "sparse_attn_ms": attn_ms,
            "sparse_attn_tflops": flops / (attn_ms * 1e-3) / 1e12,
            "sparse_attn_frac_of_bf16_peak": flops / (attn_ms * 1e-3) / 1e12 / bf16, "peak_source": src,
            "step_tflops": flops / ((mask_ms + pairing_ms + attn_ms) * 1e-3) / 1e12}


def measure_fine(args, w, p, qkv=None) -> dict:
    """Fine-grained 4-token key groups on one workload: the group mask, then the attention over the
    kept groups, on whole blocks with the other groups masked and gathered 16 groups to a tile."""
    import torch
    import dynamic_block_sparse_tile_b200 as dbst
    dbst.load()
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    to_dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()   # noqa: E731
    q, k, v = qkv if qkv is not None else (to_dev(a) for a in S.make_qkv(w))
    ws = torch.empty(dbst.fine_mask_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    mask = dbst.build_fine_mask(q, k, g, p, raster=True, workspace=ws)
    o = torch.empty_like(q)
    lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device="cuda")
    mask_ms = timed_median(lambda: dbst.build_fine_mask(q, k, g, p, raster=True, workspace=ws, out=mask),
                           args.steps, args.warmup)
    blocks_ms = timed_median(lambda: dbst.block_sparse_attn_groups(q, k, v, g, mask[1], mask[2], mask[0], raster=True,
                                                                   out=o, lse=lse), args.steps, args.warmup)
    gather_ms = timed_median(lambda: dbst.block_sparse_attn_gather(q, k, v, g, mask[0], raster=True, out=o, lse=lse),
                             args.steps, args.warmup)
    dbst.get_error()
    gm = mask[0].cpu().numpy().view(np.uint16)
    kept_groups = int(np.unpackbits(gm.view(np.uint8)).sum())
    ng = g.N // 4
    flops = 4.0 * w.D * 64 * 4 * kept_groups          # 64 queries x 4 keys per kept (query block, group)
    return {"fine": workload_desc(w, p), "kept_group_fraction": kept_groups / (g.B * g.H * g.NB * ng),
            "kept_block_fraction": int(mask[1].sum().item()) / (g.B * g.H * g.NB * g.NB), "mask_ms": mask_ms,
            "attn_whole_blocks_ms": blocks_ms, "attn_gathered_ms": gather_ms,
            "gathered_tflops_on_kept_groups": flops / (gather_ms * 1e-3) / 1e12}


def measure_dense(args, w, qkv) -> dict:
    """Dense attention from the same library on the same raster tensors (the comparator)."""
    import dynamic_block_sparse_tile_b200 as dbst
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    q, k, v = qkv
    dense_ms = timed_median(lambda: dbst.dense_attn_raster(q, k, v, g), args.steps, args.warmup)
    dbst.get_error()
    flops = 4.0 * w.D * w.N * w.N * w.B * w.H
    return {"workload": workload_desc(w, float("nan")), "dense_attn_ms": dense_ms,
            "dense_tflops": flops / (dense_ms * 1e-3) / 1e12}


def measure_squad(args) -> dict:
    """SQuad two-pass attention against dense attention on the same tensors (B=2 H=16 N=16384 D=128,
    w = sqrt(N) = 128)."""
    import torch
    import dynamic_block_sparse_tile_b200 as dbst
    dbst.load()
    w = S.workload("sweep")
    win = int(round(math.sqrt(w.N)))
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda() for a in S.make_qkv(w))
    ws = torch.empty(dbst.squad_workspace_bytes(w.B, w.H, w.N, w.D, win), dtype=torch.uint8, device="cuda")
    o = torch.empty_like(q)
    squad_ms = timed_median(lambda: dbst.squad_attn(q, k, v, win, workspace=ws, out=o), args.steps, args.warmup)
    dense_ms = timed_median(lambda: dbst.dense_attn_raster(q, k, v, g), args.steps, args.warmup)
    dbst.get_error()
    flops = 4.0 * w.D * w.N * (win + w.N // win) * w.B * w.H
    moved = 2 * 4 * w.B * w.H * w.N * w.D * 2      # four window transposes, each a read and a write
    return {"squad": f"B={w.B} H={w.H} N={w.N} D={w.D} w={win}", "squad_ms": squad_ms, "dense_attn_ms": dense_ms,
            "speedup_vs_dense": dense_ms / squad_ms, "squad_tflops": flops / (squad_ms * 1e-3) / 1e12,
            "squad_flop_fraction_of_dense": flops / (4.0 * w.D * w.N * w.N * w.B * w.H),
            "transpose_bytes": moved, "launches": 6}


def run_squad(args):
    print(json.dumps(measure_squad(args)), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="wan")
    ap.add_argument("--p", type=float, default=None)
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--ref-budget", type=float, default=0.0,
                    help="seconds of oracle work per reference step (0: about 120 s over the whole run)")
    ap.add_argument("--sweep", action="store_true",
                    help="sparsity sweep: attention ms/call and kept-block TFLOP/s per p, dense crossover")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--squad", action="store_true", help="time SQuad two-pass attention against dense attention")
    ap.add_argument("--no-extensions", action="store_true",
                    help="skip the extension measurements (backward, SIP, SQuad, the 2x4x8-tile Wan variant) "
                         "after the timed step, e.g. under a profiler's launch list")
    ap.add_argument("--fine", action="store_true",
                    help="time the 4-token key-group mask and attention (whole blocks, and gathered groups)")
    ap.add_argument("--sip", action="store_true",
                    help="time the SIP sampled mask and the attention with inclusion-probability offsets")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward (gradients over the same kept blocks) instead of the forward step")
    ap.add_argument("--path", default="fused", choices=["fused", "explicit"],
                    help="fused: tile reorder folded into the kernels (raster entry points); explicit: separate passes")
    args = ap.parse_args()
    w = S.workload(args.workload)
    p = args.p if args.p is not None else w.p_list[0]
    if args.impl == "reference":
        return run_reference(args, w, p)
    if args.sweep:
        return run_sweep(args, S.workload("sweep") if args.workload == "wan" else w)
    if args.backward:
        return run_backward(args, w, p)
    if args.squad:
        return run_squad(args)
    if args.sip:
        return run_sip(args, w, p)
    if args.fine:
        print(json.dumps(measure_fine(args, w, p)), flush=True)
        return 0

    import torch
    import torch.distributed as dist
    import dynamic_block_sparse_tile_b200 as dbst

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    dbst.load()
    g = dbst.Geom.make(w.B, w.H, w.D, w.grid, w.tile)
    q_h, k_h, v_h = S.make_qkv(w)
    to_t = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)   # noqa: E731
    host = [to_t(a).pin_memory() for a in (q_h, k_h, v_h)]
    del q_h, k_h, v_h
    q, k, v = (t.cuda() for t in host)
    o = torch.empty_like(q)
    qt = kt = vt = ot = None
    if args.path == "explicit":
        qt, kt, vt, ot = (torch.empty_like(q) for _ in range(4))
    bits = torch.empty((g.B, g.H, g.NB, g.NW), dtype=torch.int32, device="cuda")
    cnt = torch.empty((g.B, g.H, g.NB), dtype=torch.int32, device="cuda")
    idx = torch.empty((g.B, g.H, g.NB, g.NB), dtype=torch.int16, device="cuda")
    ws = torch.empty(dbst.mask_workspace_bytes(g), dtype=torch.uint8, device="cuda")
    lse = torch.empty((g.B, g.H, g.N), dtype=torch.float32, device="cuda")
    o_host = torch.empty_like(host[0]).pin_memory()
    stream = torch.cuda.current_stream()
    fused = args.path == "fused"
    # fused: 5 mask kernels + pairing + attention; explicit: 3 reorders + 5 + attention + unreorder
    launches_per_step = 7 if fused else 10   # kernels of this library (the memset is the runtime's)
    pairs = torch.empty((g.B, g.H, (g.NB + 1) // 2), dtype=torch.int32, device="cuda")

    ev = {}

    def step(timed_parts: bool, io=None):
        """One pass of the path on `stream`; io = (q, k, v, o) device buffers (default: the resident ones)."""
        q_, k_, v_, o_ = (q, k, v, o) if io is None else io
        if not fused:
            dbst.tile_reorder(q_, g, out=qt)
            dbst.tile_reorder(k_, g, out=kt)
            dbst.tile_reorder(v_, g, out=vt)
        if timed_parts:
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
        if fused:
            dbst.build_block_mask_raster(q_, k_, g, p, w.sta_radius, workspace=ws, out=(bits, cnt, idx))
        else:
            dbst.build_block_mask(qt, kt, g, p, w.sta_radius, workspace=ws, out=(bits, cnt, idx))
        if timed_parts:
            em = torch.cuda.Event(enable_timing=True)
            em.record(stream)
        if fused:
            dbst.pair_query_blocks(bits, g, out=pairs)
        if timed_parts:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(stream)
        if fused:
            dbst.block_sparse_attn_raster(q_, k_, v_, g, cnt, idx, 0.0, want_lse=True, out=o_, lse=lse, pairs=pairs)
        else:
            dbst.block_sparse_attn(qt, kt, vt, g, cnt, idx, 0.0, want_lse=True, out=ot, lse=lse)
        if timed_parts:
            e2 = torch.cuda.Event(enable_timing=True)
            e2.record(stream)
            ev.setdefault("parts", []).append((e0, e1, e2, em))
        if not fused:
            dbst.tile_unreorder(ot, g, out=o_)

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    dbst.get_error()
    kept_pairs = int(cnt.sum().item())
    kept_frac = kept_pairs / (g.B * g.H * g.NB * g.NB)
    flops = 4.0 * w.D * 64 * 64 * kept_pairs

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(args.steps):
        step(True)
    end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    dbst.get_error()
    ms_total = start.elapsed_time(end)
    mask_ms = statistics.mean(a.elapsed_time(m) for a, _, _, m in ev["parts"])      # mask build alone
    pairing_ms = statistics.mean(m.elapsed_time(b) for _, b, _, m in ev["parts"])   # query-block pairing
    attn_ms = statistics.mean(b.elapsed_time(c) for _, b, c, _ in ev["parts"])

    # End to end, as a serving loop runs it: every step copies its inputs in from pinned host
    # memory and its output back out, and the copies of neighbouring steps overlap this step's
    # compute (host->device on one stream, device->host on another; PCIe runs both directions at
    # once).  Inputs and outputs are double-buffered; events order each buffer's reuse.
    dev_io = [(q, k, v, o), tuple(torch.empty_like(q) for _ in range(4))]
    host_out = [o_host, torch.empty_like(o_host).pin_memory()]
    s_ins = [torch.cuda.Stream() for _ in range(3)]   # q, k, v copied in side by side
    s_out = torch.cuda.Stream()

    def e2e_run(n, start=None, end=None):
        ev_in, ev_done, ev_out = [[None] * 3, [None] * 3], [None, None], [None, None]
        if start is not None:
            start.record(s_ins[0])
            for s_ in s_ins[1:]:
                s_.wait_event(start)
        for i in range(n):
            b = i % 2
            for t_, (s_, src, dst) in enumerate(zip(s_ins, host, dev_io[b][:3])):
                with torch.cuda.stream(s_):
                    if ev_done[b] is not None:
                        s_.wait_event(ev_done[b])        # step i-2 has finished reading buffer b
                    dst.copy_(src, non_blocking=True)
                    ev_in[b][t_] = torch.cuda.Event()
                    ev_in[b][t_].record(s_)
            for e in ev_in[b]:
                stream.wait_event(e)
            if ev_out[b] is not None:
                stream.wait_event(ev_out[b])             # step i-2's output has left buffer b
            step(False, dev_io[b])
            ev_done[b] = torch.cuda.Event()
            ev_done[b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_done[b])
                host_out[b].copy_(dev_io[b][3], non_blocking=True)
                ev_out[b] = torch.cuda.Event()
                ev_out[b].record(s_out)
        if end is not None:
            for e in ev_out:
                if e is not None:
                    s_out.wait_event(e)
            end.record(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    barrier()
    s2 = torch.cuda.Event(enable_timing=True)
    e2 = torch.cuda.Event(enable_timing=True)
    e2e_run(args.steps, s2, e2)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = s2.elapsed_time(e2)
    dbst.get_error()

    ms_total, e2e_ms, attn_ms, mask_ms, pairing_ms = max_over_ranks([ms_total, e2e_ms, attn_ms, mask_ms, pairing_ms],
                                                                    world, "cuda")
    ms_step = ms_total / args.steps
    value = job_tflops(world, flops, ms_step)
    e2e_value = job_tflops(world, flops, e2e_ms / args.steps)

    hbm, bf16, bf16_sus, src = peaks()
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    mask_bytes = 2 * w.B * w.H * w.N * w.D * 2
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_desc(w, p), "kept_fraction": kept_frac, "kept_block_pairs": kept_pairs,
                   "l2": "inputs (385 MB per tensor) larger than L2; no flush", "parallelism": f"dp{world} (independent problems)",
                   "path": "raster in/out, tile reorder inside the kernels" if fused else
                           "explicit tile_reorder / tile_unreorder passes"},
        "sparse_attn_ms_per_call": attn_ms, "sparse_attn_tflops": attn_tflops,
        "mask_build_ms_per_call": mask_ms, "mask_build_gbs": mask_bytes / (mask_ms * 1e-3) / 1e9,
        "pairing_ms_per_call": pairing_ms,
        "roofline": {"bound": "tensor", "achieved": attn_tflops, "peak": bf16, "unit": "TFLOP/s",
                     "frac": attn_tflops / bf16, "traffic": measured_traffic(w.name, p, "raster" if fused else "tiled"),
                     "peak_source": f"{src} bf16 burst; frac of sustained {attn_tflops / bf16_sus:.3f}",
                     "frac_of_sustained": attn_tflops / bf16_sus,
                     "frac_of_nominal_dense_bf16": attn_tflops / NOMINAL_BF16_TFLOPS,
                     "kernel": "pair_attn_kernel<128, raster>" if fused else "pair_attn_kernel<128, tiled>"},
        "mask_roofline": {"bound": "hbm", "achieved": mask_bytes / (mask_ms * 1e-3) / 1e9, "peak": hbm, "unit": "GB/s",
                          "frac": mask_bytes / (mask_ms * 1e-3) / 1e9 / hbm},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "ms_per_step": e2e_ms / args.steps,
                "pipelined": "host->device of step i+1 (q, k, v on three streams) and device->host of step i-1 overlap step i",
                "h2d_bytes_per_step": 3 * host[0].numel() * 2, "d2h_bytes_per_step": o_host.numel() * 2},
        "clocks": clk, "gpu_launches": launches_per_step * args.steps,
    }
    if world == 1 and not args.no_extensions:
        # The rows built on top of the path, each timed on its own after the step above (outside its
        # timed region and launch count); a failure is recorded here and cannot touch the line.
        ext = {}
        for name, fn in (("dense_same_shape", lambda: measure_dense(args, w, (q, k, v))),
                         ("backward", lambda: measure_backward(args, w, p, (q, k, v))),
                         ("sip", lambda: measure_sip(args, w, p, (q, k, v))),
                         ("squad", lambda: measure_squad(args)),
                         ("wan_tiles_2x4x8", lambda: measure_step(args, "wan_2x4x8")),
                         ("hunyuan", lambda: measure_step(args, "hunyuan")),
                         ("sparsity_sweep", lambda: measure_sweep(args, S.workload("sweep")))):
            try:
                ext[name] = fn()
            except Exception as e:   # noqa: BLE001 - reported, not raised
                ext[name] = {"error": f"{type(e).__name__}: {e}"}
        line["extensions"] = ext
    if rank == 0 and not args.no_cpu_baseline:
        cv, cs, desc = oracle_sample(w, p, budget_s=args.cpu_budget)
        line["cpu_baseline"] = {"value": cv, "unit": "TFLOP/s", "cores": cpu_threads(), "kind": "oracle",
                                "sample": desc, "cpu_model": cpu_model(), "nproc": os.cpu_count()}
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
