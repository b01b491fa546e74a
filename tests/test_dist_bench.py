"""Multi-rank host logic of bench.py on CPU (gloo, world size 2): timing
reductions take the max over ranks, job totals sum over ranks, and every rank
draws its own independent problem."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def worker(rank, world, port, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import bench
    r, w, local = bench.dist_init(world)
    assert (r, w) == (rank, world)
    mx = bench.max_over_ranks(10.0 + rank, w)
    sm = bench.sum_over_ranks(1.0 + rank, w)
    bench.barrier(w)
    wl = bench.inputs_wl(bench.WORKLOADS[bench.WORKLOAD], r)
    out[rank] = (mx, sm, wl.seed_base)
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_reductions():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(worker, args=(world, free_port(), out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 11.0          # max over ranks
    assert out[0][1] == out[1][1] == 3.0           # sum over ranks
    assert out[0][2] != out[1][2]                  # independent problems per rank


def _bench(args, env_extra=None, timeout=600):
    import subprocess
    import sys
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR",
                                                            "MASTER_PORT")}
    env.update(env_extra or {})
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    return subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, capture_output=True, text=True,
                          timeout=timeout, env=env, cwd=root)


@pytest.mark.timeout(900)
def test_gpus_two_starts_two_ranks():
    """`bench.py --gpus 2` without a launcher starts two ranks itself (here on
    CPU with gloo, through the oracle arm on the tiny workload): the line
    reports n_gpus 2 and only rank 0 prints it."""
    import json
    r = _bench(["--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(l) for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = lines[0]
    assert line["n_gpus"] == 2 and line["impl"] == "reference"
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["value"] == line["value"] > 0
    for key in ("metric", "unit", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling", "vs_baseline",
                "dtype", "data", "config"):
        assert key in line, key
    assert line["config"]["workload"].startswith("tiny")
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


@pytest.mark.timeout(300)
def test_gpus_mismatch_refused():
    """Under a launcher whose world size differs from --gpus the run stops
    with an error instead of reporting the wrong number of GPUs."""
    r = _bench(["--gpus", "2", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "3"],
               env_extra={"WORLD_SIZE": "1", "RANK": "0", "LOCAL_RANK": "0"})
    assert r.returncode != 0
    assert "WORLD_SIZE" in r.stderr
