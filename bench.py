#!/usr/bin/env python
"""Benchmark: LVSA block-sparse attention step at the Wan-2.1-1.3B shape, 6x horizon.

One step = one pass of the LVSA hot path for one denoising step s:
  lvsa_build_index(T=126, T_per=6, W=15, C=21, s)   anchors rotate with s
  blocksparse_attn_fwd(q, k, v, frame index)          tile expansion + attention
on fresh synthetic bf16 q/k/v [N=196560, H=12, d=128] (a pool of input sets
generated before timing; every tensor is 604 MB, larger than L2, so no flush
is needed between steps).  The metric counts FLOPs on kept 128x128 tiles
(4 * d * 128 * 128 per tile and head).

Every other workload is measured in the same run at its full size and
reported as an extra key (`configs`): the tiny case, the 1x-horizon shapes
(C = 21 equal to dense, and C = 11), the balanced 6x variant, the LoSA path
on the 14B-shaped workload (dense measuring step with block mass, 99%
selection, the 39 frozen-index steps on their own perturbed inputs), the
720p 14B-head shape at all 40 heads (LVSA, LoSA alone, LoSA inside LVSA) and
the HunyuanVideo-1.5-shaped horizons with the attention path's peak memory.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {b200,reference}]
Multi-GPU: one process per GPU.  Under torchrun (WORLD_SIZE set) --gpus must
equal the world size; without a launcher and N > 1, bench.py starts the N
ranks itself through torch.distributed.run.  Each rank runs its own replica
of the workload (independent problems, no data-path collective): weak
scaling; --shard heads splits one problem by heads instead (strong scaling).
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import socket
import statistics
import subprocess
import sys
import tempfile
import time
import warnings

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_lvsa_b200.workloads import WORKLOADS  # noqa: E402
from block_sparse_attention_lvsa_b200 import inputs  # noqa: E402

METRIC = "effective TFLOP/s (kept blocks) & ms/call, Wan-1.3B shape 6x horizon; % BF16 peak"
UNIT = "TFLOP/s"
WORKLOAD = "wan1.3b_6x"
POOL = 3            # distinct fresh input sets cycled through the steps
LVSA_WORKLOADS = [n for n, w in WORKLOADS.items() if w.C is not None]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"bf16": d["bf16_tflops"], "bf16_sustained": d["bf16_tflops_sustained"],
                "hbm": d["hbm_gbs"], "src": "measured"}
    return {"bf16": 1590.0, "bf16_sustained": 1400.0, "hbm": 6650.0, "src": "fallback"}


# ------------------------------------------------------------ distributed --
def free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launch_ranks(n: int, argv) -> int:
    """Start `n` ranks of this script through torch.distributed.run (one
    process per GPU, rendezvous on 127.0.0.1) and return their exit status."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={free_port()}", os.path.abspath(__file__)] + list(argv)
    return subprocess.call(cmd)


def dist_init(n_gpus):
    """Join the process group when launched as one of several ranks; the
    world size must equal --gpus."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"--gpus {n_gpus} but WORLD_SIZE={world}: launch one rank per GPU")
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


def _reduce(x: float, world: int, op) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x: float, world: int) -> float:
    import torch.distributed as dist
    return _reduce(x, world, dist.ReduceOp.MAX if world > 1 else None)


def sum_over_ranks(x: float, world: int) -> float:
    import torch.distributed as dist
    return _reduce(x, world, dist.ReduceOp.SUM if world > 1 else None)


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
        # nvidia-smi takes a moment to start: wait (up to 5 s) for its first sample
        t0 = time.time()
        while self.proc is not None and time.time() - t0 < 5.0 and os.path.getsize(self.path) == 0:
            time.sleep(0.05)
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
CPU_ROWS_PER_HEAD = 24576     # stratified query rows per sampled head
CPU_HEADS = 2                 # heads per sample


def oracle_sample(pool, wl, step, rows_per_head, heads, seed, qkv=None):
    """Time the oracle, spread over the host cores, on a bounded sample of
    one LVSA step: `rows_per_head` stratified query rows of each of `heads`.

    Returns (seconds of the parallel oracle evaluation, kept-tile-equivalent
    FLOPs of the sample, rows).  The kept-tile-equivalent FLOPs of a row are
    the workload's kept-tile FLOPs per head-row of its query tile, so the
    rate is in the accounting of the GPU metric.
    """
    from oracle import lvsa as olvsa
    from oracle import tiles as otiles
    if qkv is None:
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        qkv = inputs.workload_qkv(wl, step, device=dev)
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, step)
    rows = inputs.sample_rows(wl.N, wl.P, rows_per_head, seed).numpy()
    work = []
    for h in heads:
        q, k, v = (x[:, h:h + 1, :].to("cpu").to(torch.float64).numpy() for x in qkv)
        work.append((pool.put_head(q, k, v), rows))
    _, dt = pool.attention_rows(work, lambda r: olvsa.allowed_keys_for_row(r, A, wl.P, wl.N),
                                lambda r: r // wl.P, wl.scale)
    pool.drop_files()
    qts = sorted(set((rows // 128).tolist()))
    idx, _ = otiles.kept_tiles(A, wl.T, wl.N, qtiles=qts)
    per_qtile = {qt: len(r) for qt, r in zip(qts, idx)}
    flops = len(heads) * sum(4 * wl.d * 128 * per_qtile[r // 128] for r in rows.tolist())
    return dt, flops, len(rows) * len(heads)


def sample_note(pool, wl):
    return (f"{CPU_HEADS} heads x {CPU_ROWS_PER_HEAD} stratified query rows (frame and tile boundaries, last "
            f"partial tile) of one LVSA step of {wl.name}, fp64 numpy oracle, {pool.workers} single-threaded "
            "worker processes over (head, query frame) tasks; kept-tile-equivalent FLOPs")


def run_reference(args, rank, world):
    """Oracle arm: the fp64 CPU oracle timed on this host's cores, on a bounded
    sample of the workload per step (rank 0 only)."""
    if rank != 0:
        return
    from oracle.pool import OraclePool
    wl = WORKLOADS[args.workload]
    pool = OraclePool()
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    rows_n = min(CPU_ROWS_PER_HEAD, wl.N)
    heads = list(range(min(CPU_HEADS, wl.H)))
    secs, flops = [], []
    try:
        for i in range(args.warmup + args.steps):
            s = i % wl.steps
            qkv = inputs.workload_qkv(wl, s, device=dev)
            dt, fl, n = oracle_sample(pool, wl, s, rows_n, [(h + s) % wl.H for h in heads], 100 + i, qkv)
            del qkv
            if i >= args.warmup:
                secs.append(dt)
                flops.append(fl)
    finally:
        workers = pool.workers
        note = sample_note(pool, wl)
        pool.close()
    value = sum(flops) / sum(secs) / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000 * sum(secs) / len(secs), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(wl, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": workers, "kind": "oracle", "sample": note},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_block(wl, world, shard="replicas", H_total=None):
    H_all = wl.H if H_total is None else H_total
    return {"workload": f"{wl.name}: LVSA block-sparse self-attention, T={wl.T} frames x P={wl.P} tokens "
                        f"(N={wl.N}), H={H_all}, d={wl.d}, C={wl.C}, W={wl.W}, T_per={wl.T_per}, anchors "
                        "rotated per step, fresh q/k/v per step",
            "N": wl.N, "H": H_all, "d": wl.d, "T": wl.T, "P": wl.P, "C": wl.C, "W": wl.W, "T_per": wl.T_per,
            "global_batch": world if shard == "replicas" else 1, "seq_len": wl.N,
            "parallelism": f"{shard} x{world}",
            "l2": "inputs larger than L2 (604 MB per tensor), no flush" if wl.N * wl.H * wl.d * 2 > 126e6
                  else "inputs smaller than L2"}


# ---------------------------------------------------------------- helpers --
def ev_timed(fn, reps, stream, warm=1):
    """Median ms of `fn` between CUDA events on `stream` over `reps` calls
    (after `warm` untimed calls)."""
    out = []
    for i in range(warm + reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        torch.cuda.synchronize()
        if i >= warm:
            out.append(a.elapsed_time(b))
    return statistics.median(out)


def graph_timed(fn, n, reps=5):
    """Median ms per call of `fn` captured `n` times into one CUDA graph (so the
    host-side cost of each call is not part of the measurement)."""
    fn()                                   # first call on the device does its set-up outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with warnings.catch_warnings():
        # a call that launches on a stream other than the capturing one leaves the graph
        # empty and its replay times nothing: make that an error, not a number
        warnings.filterwarnings("error", message=".*CUDA Graph is empty.*")
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


def rates(flop_kept, flop_exact, ms, peaks):
    """TFLOP/s on kept tiles and exact pairs, and fractions of the burst peak."""
    tk = flop_kept / (ms / 1e3) / 1e12
    te = flop_exact / (ms / 1e3) / 1e12
    return {"ms_per_call": ms, "tflops_kept_tiles": tk, "tflops_exact_pairs": te,
            "frac_of_bf16_burst": tk / peaks["bf16"], "frac_exact_of_bf16_burst": te / peaks["bf16"]}


def lvsa_tiles(bsa, wl, s, frames, counts, ws, qkv, o, lse):
    """Kept 128x128 tiles (per head) and exact allowed pairs of step s, from
    the library's own tile lists."""
    bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, frames, counts)
    ix = bsa.lvsa_index(wl.T, frames, counts)
    bsa.blocksparse_attn_fwd(*qkv, ix, scale=wl.scale, o=o, lse=lse, workspace=ws)
    _, tcnt, _, _ = bsa.lvsa_workspace_views(ws, wl.N, wl.T)
    return int(tcnt.sum().item()), int(counts.sum().item()) * wl.P * wl.P


def dense_frames(T, dev):
    f = torch.arange(T, dtype=torch.int32, device=dev).repeat(T, 1).contiguous()
    return f, torch.full((T,), T, dtype=torch.int32, device=dev)


# ------------------------------------------------------------------ main --
def run_b200(args, rank, world, local):
    from block_sparse_attention_lvsa_b200 import binding as bsa
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA GPU (the product path has no CPU fallback)")
    peaks = load_peaks()
    wl = WORKLOADS[args.workload]
    if args.heads:
        wl = dataclasses.replace(wl, H=args.heads)      # profiling case only
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream()

    # the CPU-baseline pool starts (spawn) before any GPU work of this process;
    # the baseline is taken at N = 1 only (rank 0 of a larger job would repeat it
    # while every GPU of the job waits)
    pool = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.main_only:
        from oracle.pool import OraclePool
        pool = OraclePool()

    # ---- inputs (fresh per step, cycled from a pool), outputs, index buffers
    H_total = wl.H
    if args.shard == "heads":
        # one problem split by heads: every rank draws the same inputs and keeps its head range
        from block_sparse_attention_lvsa_b200 import heads
        h0, h1 = heads.head_range(wl.H, world, rank)
        if h1 == h0:
            raise SystemExit("--shard heads needs at least as many heads as ranks")
        qpool = [tuple(heads.local_heads(x, wl.H, world, rank) for x in inputs.workload_qkv(wl, s, device=dev))
                 for s in range(POOL)]
        wl = dataclasses.replace(wl, H=h1 - h0)
    else:
        qpool = [inputs.workload_qkv(inputs_wl(wl, rank), s, device=dev) for s in range(POOL)]
    N, H, d = wl.N, wl.H, wl.d
    nB = math.ceil(N / 128)
    o = torch.empty_like(qpool[0][0])
    lse = torch.empty((H, N), dtype=torch.float32, device=dev)
    frames = torch.empty((wl.T, wl.T), dtype=torch.int32, device=dev)
    counts = torch.empty((wl.T,), dtype=torch.int32, device=dev)
    ix = bsa.lvsa_index(wl.T, frames, counts)
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, H, d, ix), dtype=torch.uint8, device=dev)

    # kept tiles and exact pairs per anchor phase (s mod T_per), from the library's own lists
    kept_tiles, exact_pairs = {}, {}
    for ph in range(wl.T_per):
        kept_tiles[ph], exact_pairs[ph] = lvsa_tiles(bsa, wl, ph, frames, counts, ws, qpool[0], o, lse)
    assert bsa.get_device_status() == bsa.BSA_OK

    def step(i, ev=None):
        s = i % wl.steps
        q, k, v = qpool[i % POOL]
        bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, frames, counts, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale, o=o, lse=lse, workspace=ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        return s

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    phases = []
    with ClockSampler(local) as clk:            # sampling covers the warm-up and the timed steps
        for i in range(args.warmup):
            step(i)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
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
    achieved_exact = sum(flop_exact) / (sum(call_ms) / 1e3) / 1e12
    clocks = clk.summary()

    if args.main_only:
        if rank == 0:
            print(json.dumps({"metric": METRIC, "value": value, "unit": UNIT, "ms_per_call": statistics.median(call_ms),
                              "tflops_kept_tiles": achieved, "heads": H, "profiling_case": True}), flush=True)
        return

    # ---- dense run of the same kernel (every tile kept), same inputs
    dframes, dcounts = dense_frames(wl.T, dev)
    dix = bsa.lvsa_index(wl.T, dframes, dcounts)
    dense_ms = ev_timed(lambda: bsa.blocksparse_attn_fwd(*qpool[1], dix, scale=wl.scale, o=o, lse=lse, workspace=ws,
                                                         stream=stream), 2, stream)
    dense_flop = 4 * d * H * nB * nB * 128 * 128
    sdpa = run_sdpa_context(qpool[0], wl.scale, stream) if rank == 0 else None
    index_us = graph_timed(lambda: bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 1, frames, counts), 50) * 1e3
    gather = run_gather(o, lse, H_total, world) if args.shard == "heads" and world > 1 else None

    # ---- e2e: host buffers through the public API, copies inside the timed region,
    # over one whole denoising run of the workload (its 40 steps)
    e2e = run_e2e(bsa, wl, qpool[0], stream, frames, counts, ix, o, lse, ws, wl.steps, kept_tiles, world)
    del qpool, o, lse, ws
    torch.cuda.empty_cache()

    # ---- every other workload at full size (N = 1 only: at N > 1 rank 0 would
    # repeat the one-GPU figures while the other GPUs of the job are held)
    configs = run_configs(bsa, stream, peaks) if world == 1 and not args.no_configs else None

    med_call = statistics.median(call_ms)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_total_ms / args.steps, "higher_is_better": True,
        "scaling": "weak" if args.shard == "replicas" else "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_block(wl, world, args.shard, H_total),
        "ms_per_call": med_call,
        "tflops_kept_tiles": achieved,
        "tflops_exact_pairs": achieved_exact,
        "frac_of_bf16_burst": achieved / peaks["bf16"],
        "speedup_vs_dense": dense_ms / med_call,
        "dense_ms_per_call": dense_ms,
        "dense_tflops": dense_flop / (dense_ms / 1e3) / 1e12,
        "kept_tile_fraction": statistics.mean(kept_tiles[ph] for ph in phases) / (nB * nB),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16"], "traffic": TRAFFIC_PER_LAUNCH,
                     "frac_exact_pairs": achieved_exact / peaks["bf16"],
                     "frac_of_sustained_peak": achieved / peaks["bf16_sustained"],
                     "peak_kind": f"bf16 dense, burst ({peaks['src']}): each ~40 ms call is timed on its own "
                                  "with CUDA events",
                     "kernel": "attn_tile_kernel<128,false> (+2 index-expansion launches of a few us in the "
                               "same call)"},
        "e2e": e2e,
        "gpu_launches": 4 * args.steps,
        "clocks": clocks,
        "lvsa_build_index": {"us": index_us, "bytes_out": (wl.T * wl.T + wl.T) * 4,
                             "note": "a few KB written: latency-bound, GB/s not meaningful"},
        "context_torch_sdpa_dense": sdpa,
        "configs": configs,
    }
    if gather is not None:
        line["gather_heads"] = gather
    if pool is not None:
        try:
            dt, fl, n = oracle_sample(pool, wl, 0, min(CPU_ROWS_PER_HEAD, wl.N), list(range(min(CPU_HEADS, wl.H))),
                                      seed=7)
            line["cpu_baseline"] = {"value": fl / dt / 1e12, "unit": UNIT, "cores": pool.workers, "kind": "oracle",
                                    "sample": sample_note(pool, wl) + f" ({dt:.1f} s)",
                                    "rows_per_s": n / dt,
                                    "extrapolated_full_call_s": dt * wl.N * H_total / n}
        finally:
            pool.close()
    if rank == 0:
        print(json.dumps(line), flush=True)


# DRAM bytes (read + write) per launch of the attention kernel at the full
# 12-head workload: the ncu capture of the 4-head case of the same workload
# (666.9 MB read + 192.4 MB written, step-0 index) scaled by 12/4 (traffic
# grows with the number of heads).  Must be re-measured (or set to None)
# whenever the kernel changes.
TRAFFIC_PER_LAUNCH = 2.578e9


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
        ms = ev_timed(lambda: F.scaled_dot_product_attention(q, k, v, scale=scale), reps, stream)
        N, H, d = qkv[0].shape
        return {"ms": ms, "tflops": 4 * d * H * N * N / (ms / 1e3) / 1e12}
    except Exception as e:                                        # noqa: BLE001 - context only
        return {"unavailable": str(e).splitlines()[0][:200]}


def inputs_wl(wl, rank):
    """Each rank draws its own independent problem (different seeds)."""
    return dataclasses.replace(wl, seed_base=wl.seed_base + 100000 * rank)


def run_e2e(bsa, wl, qkv, stream, frames, counts, ix, o, lse, ws, steps, kept_tiles, world, host_out=None):
    """Same metric through the C-ABI call with pinned host buffers, as a caller
    streaming denoising steps would run it: every step copies its q, k, v
    host -> device and its o, lse device -> host inside the timed region, on
    two copy streams that overlap the attention of the neighbouring steps
    (double-buffered device inputs and outputs, ordered by events).  The
    timed region is `steps` whole steps, the first upload (before any
    compute) and the last download (after it) included.  With `host_out` (a
    list), the pinned host copies of the last step's o and lse are appended
    to it (for checking)."""
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
    if host_out is not None:
        host_out.extend((ho, hl))
    return {"value": fl / (ms / 1e3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "ms_per_step": ms / steps, "steps": steps,
            "overlap": "copies on two streams beside the compute; first upload and last download not overlapped"}


# ------------------------------------------------------- other workloads --
def run_configs(bsa, stream, peaks):
    out = {}
    for name, fn in (("tiny", lambda: lvsa_config(bsa, "tiny", stream, peaks, steps=4, graph=True)),
                     ("wan1.3b_1x_dense", lambda: lvsa_config(bsa, "wan1.3b_1x_dense", stream, peaks, steps=5)),
                     ("wan1.3b_1x_c11", lambda: lvsa_config(bsa, "wan1.3b_1x_c11", stream, peaks, steps=5)),
                     ("wan1.3b_6x_tper21", lambda: lvsa_config(bsa, "wan1.3b_6x_tper21", stream, peaks, steps=6)),
                     ("wan14b_losa", lambda: losa_config(bsa, stream, peaks)),
                     ("720p_14b", lambda: p720_config(bsa, stream, peaks)),
                     ("hunyuan1.5_1.5x", lambda: lvsa_config(bsa, "hunyuan1.5_1.5x", stream, peaks, steps=3,
                                                             memory=True)),
                     ("hunyuan1.5_2x", lambda: lvsa_config(bsa, "hunyuan1.5_2x", stream, peaks, steps=3,
                                                           memory=True))):
        try:
            out[name] = fn()
        except Exception as e:                                    # noqa: BLE001 - reported, not hidden
            out[name] = {"error": f"{type(e).__name__}: {str(e).splitlines()[0][:200]}"}
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return out


def lvsa_config(bsa, name, stream, peaks, steps, graph=False, memory=False):
    """LVSA steps 0..steps-1 of workload `name`, each on its own inputs: ms per
    call, TFLOP/s on kept tiles and exact pairs, speed-up over the same kernel
    on a dense index; with `memory`, the attention path's peak device memory."""
    wl = WORKLOADS[name]
    N, H, d = wl.N, wl.H, wl.d
    nB = math.ceil(N / 128)
    dev = torch.device("cuda")
    if memory:
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats()
        base = torch.cuda.memory_allocated()
    frames = torch.empty((wl.T, wl.T), dtype=torch.int32, device=dev)
    counts = torch.empty((wl.T,), dtype=torch.int32, device=dev)
    ix = bsa.lvsa_index(wl.T, frames, counts)
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, H, d, ix), dtype=torch.uint8, device=dev)
    ms, kept, exact = [], 0, 0
    launch_stream = None if graph else stream      # under graph capture: the capturing (current) stream
    for s in range(steps):
        qkv = inputs.workload_qkv(wl, s, device=dev)
        o = torch.empty_like(qkv[0])
        lse = torch.empty((H, N), dtype=torch.float32, device=dev)
        kt, ep = lvsa_tiles(bsa, wl, s, frames, counts, ws, qkv, o, lse)
        kept += kt
        exact += ep
        call = lambda: bsa.blocksparse_attn_fwd(*qkv, ix, scale=wl.scale, o=o, lse=lse, workspace=ws,  # noqa: E731
                                                stream=launch_stream)
        ms.append(graph_timed(call, 20) if graph else ev_timed(call, 3, stream))
        if s < steps - 1:
            del qkv, o, lse
    peak = torch.cuda.max_memory_allocated() - base if memory else None
    dframes, dcounts = dense_frames(wl.T, dev)
    dix = bsa.lvsa_index(wl.T, dframes, dcounts)
    dcall = lambda: bsa.blocksparse_attn_fwd(*qkv, dix, scale=wl.scale, o=o, lse=lse, workspace=ws,  # noqa: E731
                                             stream=launch_stream)
    dense_ms = graph_timed(dcall, 20) if graph else ev_timed(dcall, 2, stream)
    status = bsa.get_device_status()
    mean_ms = statistics.mean(ms)
    r = rates(4 * d * H * kept * 128 * 128 / steps, 4 * d * H * exact / steps, mean_ms, peaks)
    r.update({"workload": f"T={wl.T} x P={wl.P} (N={N}), H={H}, d={d}, LVSA C={wl.C} W={wl.W} T_per={wl.T_per}, "
                          f"steps 0..{steps - 1} on their own inputs",
              "steps": steps, "kept_tile_fraction": kept / steps / (nB * nB),
              "dense_ms_per_call": dense_ms, "dense_tflops": 4 * d * H * nB * nB * 128 * 128 / (dense_ms / 1e3) / 1e12,
              "speedup_vs_dense": dense_ms / mean_ms, "status": bsa.status_string(status)})
    if graph:
        r["timing"] = "20 calls replayed from one CUDA graph per step (microsecond calls)"
    if memory:
        qkvo = 4 * N * H * d * 2
        r["memory"] = {"attention_path_peak_bytes": peak,
                       "of_which_qkvo_bytes": qkvo,
                       "workspace_bytes": ws.numel(),
                       "dense_scores_fp32_bytes_per_head": 4 * N * N,
                       "note": "peak device memory of the attention path alone (inputs, outputs, index, "
                               "workspace; torch allocator); the kernels never materialise N x N scores"}
    return r


def losa_config(bsa, stream, peaks):
    """LoSA on the Wan-2.1-14B shape: the dense measuring step with block mass
    (step 0), the 99% selection, then the 39 later steps on their own
    perturbed inputs with the frozen index; and the whole 40-step run
    against 40 dense steps of the same kernel."""
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
    t_dense = ev_timed(lambda: bsa.attn_dense_blockmass(q, k, v, 128, wl.scale, o=o, lse=lse, mass=mass,
                                                        workspace=ws, stream=stream), 3, stream)
    del ws
    # the selection runs in microseconds: time 50 launches replayed from a CUDA graph
    t_sel = graph_timed(lambda: bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt), 50)
    kept = int(cnt.sum().item())
    bix = bsa.block_index(idx, cnt)
    # dense forward alone (no mass), for the whole-run comparison
    dix = bsa.block_index(*dense_block_index(H, nB))
    t_dense_fwd = ev_timed(lambda: bsa.blocksparse_attn_fwd(q, k, v, dix, scale=wl.scale, o=o, lse=lse,
                                                            stream=stream), 2, stream)
    del q, k, v
    sparse = []
    for s in range(1, wl.steps):
        qs, ks, vs = inputs.workload_qkv(wl, s, device="cuda")
        sparse.append(ev_timed(lambda: bsa.blocksparse_attn_fwd(qs, ks, vs, bix, scale=wl.scale, o=o, lse=lse,
                                                                stream=stream), 1, stream, warm=1 if s == 1 else 0))
        del qs, ks, vs
    status = bsa.get_device_status()
    sel_bytes = mass.numel() * 4 + idx.numel() * 4 + cnt.numel() * 4
    dense_flop = 4 * d * H * N * N
    run_ms = t_dense + t_sel + sum(sparse)
    r = rates(4 * d * kept * 128 * 128, 4 * d * kept * 128 * 128, statistics.mean(sparse), peaks)
    r.pop("tflops_exact_pairs")
    r.pop("frac_exact_of_bf16_burst")
    r.update({"workload": "wan14b_losa: T=21 x P=1560 (N=32760), H=40, d=128, block 128, tau=0.99; step 0 dense "
                          "measuring step, steps 1..39 frozen index on their own perturbed inputs",
              "ms_per_call": statistics.mean(sparse), "ms_per_call_median": statistics.median(sparse),
              "frozen_steps": len(sparse),
              "dense_blockmass_ms": t_dense, "dense_blockmass_tflops_equiv": dense_flop / (t_dense / 1e3) / 1e12,
              "dense_fwd_ms": t_dense_fwd, "dense_fwd_tflops": dense_flop / (t_dense_fwd / 1e3) / 1e12,
              "select_us": t_sel * 1e3, "select_gbs": sel_bytes / (t_sel / 1e3) / 1e9,
              "select_frac_of_hbm": sel_bytes / (t_sel / 1e3) / 1e9 / peaks["hbm"],
              "kept_block_fraction": kept / (H * nB * nB),
              "run_40_steps_ms": run_ms, "dense_40_steps_ms": 40 * t_dense_fwd,
              "run_speedup_vs_dense": 40 * t_dense_fwd / run_ms,
              "status": bsa.status_string(status)})
    return r


def dense_block_index(H, nB):
    idx = torch.arange(nB, dtype=torch.int32, device="cuda").repeat(H, nB, 1).contiguous()
    cnt = torch.full((H, nB), nB, dtype=torch.int32, device="cuda")
    return idx, cnt


def p720_config(bsa, stream, peaks):
    """720p long video with 14B heads (T=63 x P=3600, all 40 heads): LVSA
    steps; LoSA alone (dense measuring step, selection, frozen-index step);
    LoSA inside LVSA (restricted measuring step, selection, intersection
    step)."""
    wl = WORKLOADS["720p_14b"]
    N, H, d = wl.N, wl.H, wl.d
    nB = math.ceil(N / 128)
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    o = torch.empty_like(q)
    lse = torch.empty((H, N), dtype=torch.float32, device="cuda")
    frames = torch.empty((wl.T, wl.T), dtype=torch.int32, device="cuda")
    counts = torch.empty((wl.T,), dtype=torch.int32, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, H, d, ix), dtype=torch.uint8, device="cuda")
    lv_ms, kept, exact = [], 0, 0
    for s in range(3):                                  # three anchor phases on the same inputs
        kt, ep = lvsa_tiles(bsa, wl, s, frames, counts, ws, (q, k, v), o, lse)
        kept += kt
        exact += ep
        lv_ms.append(ev_timed(lambda: bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale, o=o, lse=lse,
                                                               workspace=ws, stream=stream), 1, stream, warm=0))
    lvsa = rates(4 * d * H * kept * 128 * 128 / 3, 4 * d * H * exact / 3, statistics.mean(lv_ms), peaks)
    lvsa["steps"] = 3
    # LoSA inside LVSA at step 0: restricted measuring step, selection, intersection step
    bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 0, frames, counts)
    mass = torch.empty((H, nB, nB), dtype=torch.float32, device="cuda")
    wsm = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKMASS, N, H, d, ix), dtype=torch.uint8, device="cuda")
    t_rmass = ev_timed(lambda: bsa.attn_blockmass(q, k, v, ix, wl.scale, o=o, lse=lse, mass=mass, workspace=wsm,
                                                  stream=stream), 1, stream)
    idx = torch.empty((H, nB, nB), dtype=torch.int32, device="cuda")
    cnt = torch.empty((H, nB), dtype=torch.int32, device="cuda")
    t_sel_r = graph_timed(lambda: bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt), 5)
    kept_r = int(cnt.sum().item())
    lvsa0_tiles = lvsa_tiles(bsa, wl, 0, frames, counts, ws, (q, k, v), o, lse)[0]
    ix3 = bsa.lvsa_block_index(wl.T, frames, counts, idx, cnt)
    ws3 = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, H, d, ix3), dtype=torch.uint8,
                      device="cuda")
    t_both = ev_timed(lambda: bsa.blocksparse_attn_fwd(q, k, v, ix3, scale=wl.scale, o=o, lse=lse, workspace=ws3,
                                                       stream=stream), 2, stream)
    del ws3
    # LoSA alone on the same inputs: dense measuring step (head passes in a 4 GiB workspace), selection, sparse step
    t_dmass = ev_timed(lambda: bsa.attn_dense_blockmass(q, k, v, 128, wl.scale, o=o, lse=lse, mass=mass,
                                                        workspace=wsm, stream=stream), 1, stream)
    del wsm
    t_sel = graph_timed(lambda: bsa.losa_select(mass, wl.tau, idx=idx, cnt=cnt), 5)
    kept_l = int(cnt.sum().item())
    bix = bsa.block_index(idx, cnt)
    t_losa = ev_timed(lambda: bsa.blocksparse_attn_fwd(q, k, v, bix, scale=wl.scale, o=o, lse=lse, stream=stream),
                      2, stream)
    status = bsa.get_device_status()
    sel_bytes = mass.numel() * 8 + cnt.numel() * 4
    fl = lambda tiles: 4 * d * tiles * 128 * 128                  # noqa: E731
    dense_flop = 4 * d * H * N * N
    return {"workload": f"720p_14b: T=63 x P=3600 (N={N}), H={H}, d=128, LVSA C=21 W=15 T_per=6; LoSA tau=0.99",
            "lvsa": lvsa,
            "losa_in_lvsa": {"restricted_mass_ms": t_rmass, "select_us": t_sel_r * 1e3,
                             "select_gbs": sel_bytes / (t_sel_r / 1e3) / 1e9,
                             "intersection_ms": t_both,
                             "intersection_tflops_kept_tiles": fl(kept_r) / (t_both / 1e3) / 1e12,
                             "kept_fraction_of_lvsa_tiles": kept_r / (lvsa0_tiles * H)},
            "losa": {"dense_blockmass_ms": t_dmass, "dense_blockmass_tflops_equiv": dense_flop / (t_dmass / 1e3) / 1e12,
                     "select_us": t_sel * 1e3, "select_gbs": sel_bytes / (t_sel / 1e3) / 1e9,
                     "sparse_ms": t_losa, "sparse_tflops_kept_blocks": fl(kept_l) / (t_losa / 1e3) / 1e12,
                     "kept_block_fraction": kept_l / (H * nB * nB)},
            "status": bsa.status_string(status)}


def run_select_only():
    """Profiling case for the LoSA selection alone, small on the device: block
    masses from a 4-head dense measuring step on the Wan-2.1-14B shape, tiled
    to that workload's 40 heads (10,240 rows of 256 key blocks)."""
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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", choices=LVSA_WORKLOADS, default=WORKLOAD,
                    help="LVSA workload of the timed steps (default: the headline 6x-horizon shape)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' extra keys")
    ap.add_argument("--heads", type=int, default=0, help="profiling only: override the head count")
    ap.add_argument("--main-only", action="store_true", help="profiling only: timed LVSA steps, nothing else")
    ap.add_argument("--select-only", action="store_true", help="profiling only: the LoSA selection, small case")
    ap.add_argument("--shard", choices=["replicas", "heads"], default="replicas",
                    help="N > 1: independent replicas (weak scaling) or one problem split by heads (strong)")
    argv = sys.argv[1:] if argv is None else argv
    args = ap.parse_args(argv)
    if args.select_only:
        run_select_only()
        return 0
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    if args.gpus < 1:
        raise SystemExit("--gpus must be >= 1")
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        return launch_ranks(args.gpus, argv)
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
    return 0


if __name__ == "__main__":
    sys.exit(main())
