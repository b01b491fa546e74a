#!/usr/bin/env python
"""Benchmark: LVSA block-sparse attention step at the Wan-2.1-1.3B shape, 6x horizon.

One step = one pass of the LVSA hot path for one denoising step s:
  lvsa_build_index(T=126, T_per=6, W=15, C=21, s)   anchors rotate with s
  blocksparse_attn_fwd(q, k, v, frame index)          tile expansion + attention
on fresh synthetic bf16 q/k/v [N=196560, H=12, d=128] (a pool of input sets
generated before timing; every tensor is 604 MB, larger than L2, so no flush
is needed between steps).  The metric counts FLOPs on kept 128x128 tiles
(4 * d * 128 * 128 per tile and head).

Also measured in the same run (reported as extra keys): the same kernel run
dense (every tile), the exact-pair FLOP rate, and the LoSA path on the
14B-shaped workload (dense measuring step with block mass, 99% selection,
frozen-index sparse steps).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {b200,reference}]
Multi-GPU: launched by torchrun; each rank runs its own replica of the
workload (independent problems, no data-path collective): weak scaling.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_lvsa_b200.workloads import WORKLOADS  # noqa: E402
from block_sparse_attention_lvsa_b200 import inputs  # noqa: E402

METRIC = "effective TFLOP/s (kept blocks) & ms/call, Wan-1.3B shape 6x horizon; % BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = "wan1.3b_6x"
POOL = 3            # distinct fresh input sets cycled through the steps


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "hbm": d["hbm_gbs"], "src": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "src": "fallback"}


# ------------------------------------------------------------ distributed --
def dist_init(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------- clocks --
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, mx, reasons, power = [], None, set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx = float(parts[2])
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for nm, val in zip(names, parts[5:9]):
                    if val.lower().startswith("active"):
                        reasons.add(nm)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": ["no samples"]}
        busy = [x for x in sm if x > 0.5 * (mx or max(sm))] or sm
        return {"sm_mhz": statistics.median(busy), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w_max": max(power) if power else None}


# ---------------------------------------------------------- CPU baseline --
def oracle_sample(wl, step, rows_n, head, qkv=None, seed=0):
    """Time the oracle on a bounded sample: ``rows_n`` query rows of one head.

    Returns (seconds, kept-tile-equivalent FLOPs of the sample, rows, cores).
    The kept-tile-equivalent FLOPs are the workload's kept-tile FLOPs per
    head-row times the number of sampled rows, so the rate is in the same
    accounting as the GPU metric.
    """
    import numpy as np
    from oracle import attention as oatt
    from oracle import lvsa as olvsa
    from oracle import tiles as otiles
    if qkv is None:
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        qkv = inputs.workload_qkv(wl, step, device=dev)
    q, k, v = (x[:, head:head + 1, :].to("cpu").to(torch.float64).numpy() for x in qkv)
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, step)
    rows = inputs.sample_rows(wl.N, wl.P, rows_n, seed).numpy()
    t0 = time.perf_counter()
    oatt.attention_rows(q, k, v, wl.scale, rows, [0],
                        lambda h, r: olvsa.allowed_keys_for_row(r, A, wl.P, wl.N),
                        lambda h, r: r // wl.P)
    dt = time.perf_counter() - t0
    idx, _ = otiles.kept_tiles(A, wl.T, wl.N, qtiles=sorted(set((rows // 128).tolist())))
    per_qtile = {qt: len(r) for qt, r in zip(sorted(set((rows // 128).tolist())), idx)}
    flops = sum(4 * wl.d * 128 * per_qtile[r // 128] for r in rows)   # kept-tile FLOPs per row
    cores = len(os.sched_getaffinity(0))
    return dt, flops, len(rows), cores


def run_reference(args, rank, world):
    """Oracle arm: the fp64 CPU oracle timed on this host's cores."""
    if rank != 0:
        return
    wl = WORKLOADS[WORKLOAD]
    rows_n = 48
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    secs, flops = [], []
    cores = len(os.sched_getaffinity(0))
    for i in range(args.warmup + args.steps):
        s = i % wl.steps
        qkv = inputs.workload_qkv(wl, s, device=dev)
        dt, fl, n, cores = oracle_sample(wl, s, rows_n, head=s % wl.H, qkv=qkv, seed=100 + i)
        del qkv
        if i >= args.warmup:
            secs.append(dt)
            flops.append(fl)
    value = sum(flops) / sum(secs) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * sum(secs) / len(secs), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(wl, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": f"{rows_n} query rows of one head per step (stratified), fp64 numpy, "
                                       "value in kept-tile-equivalent FLOPs"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_block(wl, world, shard="replicas", H_total=None):
    H_all = wl.H if H_total is None else H_total
    return {"workload": f"{wl.name}: LVSA block-sparse self-attention, Wan-2.1-1.3B shape at 6x horizon, "
                        f"T={wl.T} frames x P={wl.P} tokens (N={wl.N}), H={H_all}, d={wl.d}, "
                        f"C={wl.C}, W={wl.W}, T_per={wl.T_per}, anchors rotated per step, fresh q/k/v per step",
            "N": wl.N, "H": H_all, "d": wl.d, "T": wl.T, "P": wl.P, "C": wl.C, "W": wl.W, "T_per": wl.T_per,
            "global_batch": world if shard == "replicas" else 1, "seq_len": wl.N,
            "parallelism": f"{shard} x{world}",
            "l2": "inputs larger than L2 (604 MB per tensor), no flush"}


# ------------------------------------------------------------------ main --
def run_b200(args, rank, world, local):
    from block_sparse_attention_lvsa_b200 import binding as bsa
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the product path has no CPU fallback)")
    peaks = load_peaks()
    wl = WORKLOADS[WORKLOAD]
    if args.heads:
        import dataclasses
        wl = dataclasses.replace(wl, H=args.heads)      # profiling case only
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()
    N, H, d = wl.N, wl.H, wl.d
    nB = math.ceil(N / 128)

    # ---- inputs (fresh per step, cycled from a pool), outputs, index buffers
    H_total = wl.H
    if args.shard == "heads":
        # one problem split by heads: every rank draws the same inputs and keeps its head range
        from block_sparse_attention_lvsa_b200 import heads
        import dataclasses
        h0, h1 = heads.head_range(wl.H, world, rank)
        if h1 == h0:
            raise SystemExit("--shard heads needs at least as many heads as ranks")
        pool = [tuple(heads.local_heads(x, wl.H, world, rank) for x in inputs.workload_qkv(wl, s, device=dev))
                for s in range(POOL)]
        wl = dataclasses.replace(wl, H=h1 - h0)
        H = wl.H
    else:
        pool = [inputs.workload_qkv(inputs_wl(wl, rank), s, device=dev) for s in range(POOL)]
    o = torch.empty_like(pool[0][0])
    lse = torch.empty((H, N), dtype=torch.float32, device=dev)
    frames = torch.empty((wl.T, wl.T), dtype=torch.int32, device=dev)
    counts = torch.empty((wl.T,), dtype=torch.int32, device=dev)
    ix = bsa.lvsa_index(wl.T, frames, counts)
    ws_bytes = bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, H, d, ix)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    # kept tiles and exact pairs per anchor phase (s mod T_per), from the library's own lists
    kept_tiles, exact_pairs = {}, {}
    for ph in range(wl.T_per):
        bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, ph, frames, counts)
        bsa.blocksparse_attn_fwd(*pool[0], ix, scale=wl.scale, o=o, lse=lse, workspace=ws)
        _, tcnt, _, _ = bsa.lvsa_workspace_views(ws, N, wl.T)
        kept_tiles[ph] = int(tcnt.sum().item())
        exact_pairs[ph] = int(counts.sum().item()) * wl.P * wl.P
    assert bsa.get_device_status() == bsa.BSA_OK

    def step(i, ev=None):
        s = i % wl.steps
        q, k, v = pool[i % POOL]
        bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, frames, counts, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale, o=o, lse=lse, workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        return s

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    phases = []
    with ClockSampler(local) as clk:
        t_start.record(stream)
        for i in range(args.steps):
            phases.append(step(args.warmup + i, evs[i]) % wl.T_per)
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    status = bsa.get_device_status()
    if status != bsa.BSA_OK:
        raise SystemExit(f"device status {bsa.status_string(status)} after the timed region")
    total_ms = t_start.elapsed_time(t_end)
    call_ms = [a.elapsed_time(b) for a, b in evs]
    max_total_ms = max_over_ranks(total_ms, world)
    flop_tile = [4 * d * H * kept_tiles[ph] * 128 * 128 for ph in phases]
    flop_exact = [4 * d * H * exact_pairs[ph] for ph in phases]
    job_flop = sum_over_ranks(float(sum(flop_tile)), world)
    value = job_flop / (max_total_ms / 1e3) / 1e12
    achieved = sum(flop_tile) / (sum(call_ms) / 1e3) / 1e12          # per-launch, this rank
    clocks = clk.summary()

    if args.main_only:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "ms_per_call": statistics.median(call_ms),
                              "tflops_kept_tiles": achieved, "heads": H, "profiling_case": True}), flush=True)
        return

    # ---- dense run of the same kernel (every tile kept), same inputs
    dframes = torch.arange(wl.T, dtype=torch.int32, device=dev).repeat(wl.T, 1).contiguous()
    dcounts = torch.full((wl.T,), wl.T, dtype=torch.int32, device=dev)
    dix = bsa.lvsa_index(wl.T, dframes, dcounts)
    dense_ms = []
    for i in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        bsa.blocksparse_attn_fwd(*pool[i % POOL], dix, scale=wl.scale, o=o, lse=lse, workspace=ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            dense_ms.append(a.elapsed_time(b))
    dense_ms = statistics.median(dense_ms)
    dense_flop = 4 * d * H * nB * nB * 128 * 128
    sdpa = run_sdpa_context(pool[0], wl.scale, stream) if rank == 0 else None
    index_us = graph_timed(lambda: bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 1, frames, counts), 50) * 1e3

    # ---- balanced variant of the same shape (T_per = 21: |A(t)| = C = 21 for every t and s)
    balanced = run_balanced(bsa, pool, stream, frames, counts, ix, o, lse, ws) if rank == 0 else None
    gather = run_gather(o, lse, H_total, world) if args.shard == "heads" and world > 1 else None

    # ---- e2e: host buffers through the public API, copies inside the timed region,
    # over one whole denoising run of the workload (its 40 steps)
    e2e = run_e2e(bsa, wl, pool[0], stream, frames, counts, ix, o, lse, ws, wl.steps, kept_tiles, world)
    del pool

    # ---- LoSA path on the 14B-shaped workload, and LoSA inside LVSA at 720p (secondary)
    losa = run_losa(bsa, rank, stream, peaks) if rank == 0 else None
    lvsa_losa = run_lvsa_losa(bsa, stream) if rank == 0 else None

    med_call = statistics.median(call_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak" if args.shard == "replicas" else "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_block(wl, world, args.shard, H_total),
        "ms_per_call": med_call,
        "tflops_kept_tiles": achieved,
        "tflops_exact_pairs": sum(flop_exact) / (sum(call_ms) / 1e3) / 1e12,
        "frac_of_bf16_burst": achieved / peaks["bf16"],
        "speedup_vs_dense": dense_ms / med_call,
        "dense_ms_per_call": dense_ms,
        "dense_tflops": dense_flop / (dense_ms / 1e3) / 1e12,
        "kept_tile_fraction": statistics.mean(kept_tiles[ph] for ph in phases) / (nB * nB),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_sustained"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_sustained"], "traffic": TRAFFIC_PER_LAUNCH,
                     "peak_kind": f"bf16 dense, sustained ({peaks['src']}); kernel timed inside back-to-back steps",
                     "kernel": "attn_tile_kernel<128,false> (+2 index-expansion launches of a few us in the same call)"},
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "losa": losa,
        "balanced_tper21": balanced,
        "losa_within_lvsa_720p": lvsa_losa,
        "lvsa_build_index": {"us": index_us, "bytes_out": (wl.T * wl.T + wl.T) * 4,
                             "note": "a few KB written: latency-bound, GB/s not meaningful"},
        "context_torch_sdpa_dense": sdpa,
    }
    if gather is not None:
        line["gather_heads"] = gather
    if rank == 0 and not args.no_cpu_baseline:
        dt, fl, n, cores = oracle_sample(wl, 0, args.cpu_rows, head=0, qkv=None, seed=7)
        line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": f"{n} stratified query rows of head 0 at step 0 ({dt:.1f} s), fp64 numpy; "
                                          "kept-tile-equivalent FLOPs",
                                "rows_per_s": n / dt,
                                "extrapolated_full_call_s": dt * wl.N * H_total / n}
    if rank == 0:
        print(json.dumps(line), flush=True)


# DRAM bytes (read + write) per launch of the attention kernel at the full
# 12-head workload: the ncu capture of the 4-head case of the same workload
# (658.5 MB read + 190.7 MB written, step-0 index) scaled by 12/4 - traffic
# grows with the number of heads.  Must be re-measured (or set to None)
# whenever the kernel changes.
TRAFFIC_PER_LAUNCH = 2.548e9


def run_gather(o, lse, H, world, reps=3):
    """Time of assembling every rank's O and LSE shards on all ranks (one
    all-gather per tensor; NCCL over NVLink), outside the attention path."""
    from block_sparse_attention_lvsa_b200 import heads
    ms = []
    for i in range(reps + 1):
        barrier(world)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        og, lg = heads.gather_heads(o, lse, H)
        b.record()
        torch.cuda.synchronize()
        if i:
            ms.append(max_over_ranks(a.elapsed_time(b), world))
    nbytes = og.numel() * og.element_size() + lg.numel() * lg.element_size()
    return {"ms": statistics.median(ms), "bytes_per_rank_out": nbytes,
            "note": "not part of the timed steps; the path itself has no exchange"}


def run_sdpa_context(qkv, scale, stream, reps=2):
    """Context only (a library kernel, not part of this path): torch's
    scaled_dot_product_attention, dense, on the same q, k, v."""
    import torch.nn.functional as F
    q, k, v = (x.transpose(0, 1).unsqueeze(0) for x in qkv)       # [1, H, N, d] views
    try:
        ms = []
        for i in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            out = F.scaled_dot_product_attention(q, k, v, scale=scale)
            b.record(stream)
            torch.cuda.synchronize()
            if i:
                ms.append(a.elapsed_time(b))
        del out
        N, H, d = qkv[0].shape
        return {"ms": statistics.median(ms), "tflops": 4 * d * H * N * N / (statistics.median(ms) / 1e3) / 1e12}
    except Exception as e:                                        # noqa: BLE001 - context only
        return {"unavailable": str(e).splitlines()[0][:200]}


def run_lvsa_losa(bsa, stream, heads=4):
    """LoSA's selection inside LVSA's frame sets on the 720p Wan-14B shape
    (T=63 x P=3600, d=128), `heads` of its 40 heads: the restricted measuring
    step (LVSA attention + block mass), the selection, and a later step on
    the intersection index against LVSA alone.  Times scale with heads."""
    import dataclasses
    wl = dataclasses.replace(WORKLOADS["720p_14b"], H=heads)
    N, H, d, nB = wl.N, wl.H, wl.d, math.ceil(wl.N / 128)
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 0, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    o = torch.empty_like(q)
    lse = torch.empty((H, N), dtype=torch.float32, device="cuda")
    mass = torch.empty((H, nB, nB), dtype=torch.float32, device="cuda")
    ws_m = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKMASS, N, H, d, ix), dtype=torch.uint8, device="cuda")

    def timed(fn, reps=2):
        out = []
        for i in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            if i:
                out.append(a.elapsed_time(b))
        return statistics.median(out)

    t_mass = timed(lambda: bsa.attn_blockmass(q, k, v, ix, wl.scale, o=o, lse=lse, mass=mass, workspace=ws_m,
                                              stream=stream))
    del ws_m
    idx, cnt = bsa.losa_select(mass, wl.tau)
    t_sel = graph_timed(lambda: bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt), 10)
    ix3 = bsa.lvsa_block_index(wl.T, frames, counts, idx, cnt)
    ws_f = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, H, d, ix3), dtype=torch.uint8,
                       device="cuda")
    t_lvsa = timed(lambda: bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale, o=o, lse=lse, workspace=ws_f,
                                                    stream=stream))
    _, tcnt, _, _ = bsa.lvsa_workspace_views(ws_f, N, wl.T)
    lvsa_tiles = int(tcnt.sum().item()) * H
    t_both = timed(lambda: bsa.blocksparse_attn_fwd(q, k, v, ix3, scale=wl.scale, o=o, lse=lse, workspace=ws_f,
                                                    stream=stream))
    status = bsa.get_device_status()
    kept = int(cnt.sum().item())
    flop = lambda tiles: 4 * d * tiles * 128 * 128               # noqa: E731
    return {"workload": f"720p_14b: T=63 x P=3600 (N={N}), {H} of 40 heads, d=128, LVSA C=21 W=15 T_per=6, "
                        "LoSA tau=0.99 inside the LVSA sets",
            "restricted_mass_ms": t_mass, "select_us": t_sel * 1e3,
            "lvsa_ms": t_lvsa, "lvsa_tflops_kept_tiles": flop(lvsa_tiles) / (t_lvsa / 1e3) / 1e12,
            "intersection_ms": t_both, "intersection_tflops_kept_tiles": flop(kept) / (t_both / 1e3) / 1e12,
            "kept_fraction_of_lvsa_tiles": kept / lvsa_tiles, "status": bsa.status_string(status)}


def run_balanced(bsa, pool, stream, frames, counts, ix, o, lse, ws, calls=6):
    """The balanced reading of the 6x-horizon shape (T_per = 21, 6 anchors +
    15 window frames = C): ms per call and TFLOP/s on kept tiles over the
    first `calls` steps (anchor phases 0..calls-1), each on its own inputs."""
    wl = WORKLOADS["wan1.3b_6x_tper21"]
    ms, flop, kept = [], 0, 0
    for s in range(calls + 1):
        bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, frames, counts, stream=stream)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        bsa.blocksparse_attn_fwd(*pool[s % len(pool)], ix, scale=wl.scale, o=o, lse=lse, workspace=ws, stream=stream)
        b.record(stream)
        torch.cuda.synchronize()
        if s == 0:
            continue                                  # warm-up for this index shape
        _, tcnt, _, _ = bsa.lvsa_workspace_views(ws, wl.N, wl.T)
        k = int(tcnt.sum().item())
        kept += k
        flop += 4 * wl.d * pool[0][0].shape[1] * k * 128 * 128
        ms.append(a.elapsed_time(b))
    status = bsa.get_device_status()
    nB = math.ceil(wl.N / 128)
    return {"workload": "wan1.3b_6x_tper21: as the headline shape with T_per=21 (|A(t)| = C = 21 for every t, s)",
            "ms_per_call": statistics.median(ms), "tflops_kept_tiles": flop / (sum(ms) / 1e3) / 1e12,
            "kept_tile_fraction": kept / calls / (nB * nB), "steps": calls, "status": bsa.status_string(status)}


def inputs_wl(wl, rank):
    """Each rank draws its own independent problem (different seeds)."""
    import dataclasses
    return dataclasses.replace(wl, seed_base=wl.seed_base + 100000 * rank)


def run_e2e(bsa, wl, qkv, stream, frames, counts, ix, o, lse, ws, steps, kept_tiles, world):
    """Same metric through the C-ABI call with pinned host buffers, as a caller
    streaming denoising steps would run it: every step copies its q, k, v
    host -> device and its o, lse device -> host inside the timed region, on
    two copy streams that overlap the attention of the neighbouring steps
    (double-buffered device inputs and outputs, ordered by events).  The
    timed region is `steps` whole steps, the first upload (before any
    compute) and the last download (after it) included."""
    hq, hk, hv = (x.to("cpu").pin_memory() for x in qkv)
    ho = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    hl = torch.empty(lse.shape, dtype=lse.dtype, pin_memory=True)
    din = [tuple(torch.empty_like(x) for x in qkv) for _ in range(2)]
    dout = [(o, lse), (torch.empty_like(o), torch.empty_like(lse))]
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = ho.numel() * ho.element_size() + hl.numel() * hl.element_size()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n):
        ev = lambda: torch.cuda.Event()   # noqa: E731
        uploaded, computed, downloaded = [], [], []
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(stream)
        up.wait_event(start)
        down.wait_event(start)
        for s in range(n):
            b = s % 2
            with torch.cuda.stream(up):                 # inputs of step s into buffer b
                if s >= 2:
                    up.wait_event(computed[s - 2])      # buffer b read by step s-2
                for dst, src in zip(din[b], (hq, hk, hv)):
                    dst.copy_(src, non_blocking=True)
                uploaded.append(ev())
                uploaded[s].record(up)
            stream.wait_event(uploaded[s])
            if s >= 2:
                stream.wait_event(downloaded[s - 2])    # output buffer b copied out
            bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, frames, counts, stream=stream)
            bsa.blocksparse_attn_fwd(*din[b], ix, scale=wl.scale, o=dout[b][0], lse=dout[b][1], workspace=ws,
                                     stream=stream)
            computed.append(ev())
            computed[s].record(stream)
            with torch.cuda.stream(down):               # results of step s to the host
                down.wait_event(computed[s])
                ho.copy_(dout[b][0], non_blocking=True)
                hl.copy_(dout[b][1], non_blocking=True)
                downloaded.append(ev())
                downloaded[s].record(down)
        stream.wait_event(downloaded[n - 1])
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end)

    run(2)                                              # warm-up
    barrier(world)
    ms = max_over_ranks(run(steps), world)
    fl = sum_over_ranks(float(sum(4 * wl.d * wl.H * kept_tiles[s % wl.T_per] * 128 * 128 for s in range(steps))),
                        world)
    return {"value": fl / (ms / 1e3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / steps, "steps": steps,
            "overlap": "copies on two streams beside the compute; first upload and last download not overlapped"}


def graph_timed(fn, n, reps=5):
    """Median ms per call of `fn` captured `n` times into one CUDA graph (so the
    host-side cost of each call is not part of the measurement)."""
    fn()                                   # first call on the device does its set-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for _ in range(n):
                fn()
    out = []
    for i in range(reps + 1):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        if i:
            out.append(a.elapsed_time(b) / n)
    del g
    return statistics.median(out)


def run_losa(bsa, rank, stream, peaks):
    """LoSA on the Wan-2.1-14B shape: dense measuring step + mass, selection, frozen reuse."""
    wl = WORKLOADS["wan14b_losa"]
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    N, H, d = wl.N, wl.H, wl.d
    nB = math.ceil(N / 128)
    o = torch.empty_like(q)
    lse = torch.empty((H, N), dtype=torch.float32, device="cuda")
    mass = torch.empty((H, nB, nB), dtype=torch.float32, device="cuda")
    idx = torch.empty((H, nB, nB), dtype=torch.int32, device="cuda")
    cnt = torch.empty((H, nB), dtype=torch.int32, device="cuda")
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_DENSE_BLOCKMASS, N, H, d), dtype=torch.uint8, device="cuda")

    def timed(fn, reps, batch=1):
        """Median ms per call; `batch` calls run back to back between the events
        (for microsecond kernels, so host-side call overhead is not timed)."""
        out = []
        for i in range(reps + 1):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(batch):
                fn()
            b.record(stream)
            torch.cuda.synchronize()
            if i:
                out.append(a.elapsed_time(b) / batch)
        return statistics.median(out)

    t_dense = timed(lambda: bsa.attn_dense_blockmass(q, k, v, 128, wl.scale, o=o, lse=lse, mass=mass,
                                                     workspace=ws, stream=stream), 3)
    # the selection runs in microseconds: time 50 launches replayed from a CUDA graph
    t_sel = graph_timed(lambda: bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt), 50)
    kept = int(cnt.sum().item())
    bix = bsa.block_index(idx, cnt)
    qs = [inputs.workload_qkv(wl, s, device="cuda") for s in (1, 2)]
    t_sparse = timed(lambda: bsa.blocksparse_attn_fwd(*qs[0], bix, scale=wl.scale, o=o, lse=lse, stream=stream), 5)
    status = bsa.get_device_status()
    dense_flop = 4 * d * H * N * N
    sel_bytes = mass.numel() * 4 + idx.numel() * 4 + cnt.numel() * 4
    return {"workload": "wan14b_losa: T=21 x P=1560 (N=32760), H=40, d=128, block 128, tau=0.99",
            "dense_blockmass_ms": t_dense,
            "dense_fwd_tflops_equiv": dense_flop / (t_dense / 1e3) / 1e12,
            "select_us": t_sel * 1e3, "select_gbs": sel_bytes / (t_sel / 1e3) / 1e9,
            "select_frac_of_hbm": sel_bytes / (t_sel / 1e3) / 1e9 / peaks["hbm"],
            "kept_block_fraction": kept / (H * nB * nB),
            "sparse_ms_per_call": t_sparse,
            "sparse_tflops_kept_blocks": 4 * d * kept * 128 * 128 / (t_sparse / 1e3) / 1e12,
            "status": bsa.status_string(status)}


def run_select_only():
    """Profiling case for the LoSA selection alone, small on the device: block
    masses from a 4-head dense measuring step on the Wan-2.1-14B shape, tiled
    to that workload's 40 heads (10,240 rows of 256 key blocks)."""
    import dataclasses
    import block_sparse_attention_lvsa_b200.binding as bsa
    wl = dataclasses.replace(WORKLOADS["wan14b_losa"], H=4)
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    _, _, mass4 = bsa.attn_dense_blockmass(q, k, v, 128, wl.scale)
    del q, k, v
    mass = mass4.repeat(10, 1, 1).contiguous()
    idx, cnt = bsa.losa_select(mass, wl.tau)
    for _ in range(3):
        bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt)
    b.record()
    torch.cuda.synchronize()
    print(json.dumps({"profile": "losa_select", "rows": mass.shape[0] * mass.shape[1], "nKB": mass.shape[2],
                      "us": a.elapsed_time(b) * 1e3, "status": bsa.status_string(bsa.get_device_status())}))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--cpu-rows", type=int, default=16384)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--heads", type=int, default=0, help="profiling only: override the head count")
    ap.add_argument("--main-only", action="store_true", help="profiling only: timed LVSA steps, nothing else")
    ap.add_argument("--select-only", action="store_true", help="profiling only: the LoSA selection, small case")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: independent replicas (weak scaling) or one problem split by heads (strong)")
    args = ap.parse_args()
    if args.select_only:
        run_select_only()
        return
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    rank, world, local = dist_init(args.gpus)
    try:
        if args.impl == "reference":
            run_reference(args, rank, world)
        else:
            run_b200(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
