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
