"""Head sharding across ranks (CPU, gloo): the head split covers every head
once, gather_heads reassembles O and LSE exactly for uneven head counts, and
attention computed per rank on its heads equals attention on all heads (the
oracle on the tiny LVSA workload)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_attention_lvsa_b200 import heads


def free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


@pytest.mark.parametrize("H", range(1, 14))
@pytest.mark.parametrize("world", range(1, 6))
def test_head_range_partition(H, world):
    seen = []
    sizes = []
    for r in range(world):
        h0, h1 = heads.head_range(H, world, r)
        assert 0 <= h0 <= h1 <= H
        seen.extend(range(h0, h1))
        sizes.append(h1 - h0)
    assert seen == list(range(H))                   # contiguous, disjoint, complete, in rank order
    assert max(sizes) - min(sizes) <= 1
    assert sizes == sorted(sizes, reverse=True)     # larger shares first


def full_tensors(H, N=40, d=8):
    g = torch.Generator().manual_seed(H)
    o = torch.randn((N, H, d), generator=g).to(torch.bfloat16)
    lse = torch.randn((H, N), generator=g)
    return o, lse


def gather_worker(rank, world, port, H, out):
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    o, lse = full_tensors(H)
    o_loc = heads.local_heads(o, H, world, rank, head_dim=1)
    l_loc = heads.local_heads(lse, H, world, rank, head_dim=0)
    og, lg = heads.gather_heads(o_loc, l_loc, H)
    out[rank] = bool(torch.equal(og, o) and torch.equal(lg, lse))
    dist.destroy_process_group()


@pytest.mark.timeout(120)
@pytest.mark.parametrize("world,H", [(2, 5), (3, 5), (3, 12)])
def test_gather_heads_exact(world, H):
    out = mp.Manager().dict()
    mp.spawn(gather_worker, args=(world, free_port(), H, out), nprocs=world, join=True)
    assert all(out[r] for r in range(world))


def attention_worker(rank, world, port, out):
    from oracle import attention as oatt, lvsa as olvsa
    from block_sparse_attention_lvsa_b200 import inputs
    from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
    import dataclasses
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    wl = dataclasses.replace(WORKLOADS["tiny"], H=3)
    q, k, v = inputs.workload_qkv(wl, 1)
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, 1)
    mask = olvsa.dense_token_mask(A, wl.P, wl.N)

    def attend(qh, kh, vh):
        O, L = oatt.attention_dense_masked(qh.double().numpy(), kh.double().numpy(), vh.double().numpy(),
                                           wl.scale, mask)
        return torch.from_numpy(O), torch.from_numpy(L)

    O_loc, L_loc = attend(*(heads.local_heads(x, wl.H, world, rank) for x in (q, k, v)))
    Og, Lg = heads.gather_heads(O_loc, L_loc, wl.H)
    O_all, L_all = attend(q, k, v)
    out[rank] = bool(torch.equal(Og, O_all) and torch.equal(Lg, L_all))
    dist.destroy_process_group()


@pytest.mark.timeout(180)
def test_sharded_attention_equals_unsharded():
    world = 2
    out = mp.Manager().dict()
    mp.spawn(attention_worker, args=(world, free_port(), out), nprocs=world, join=True)
    assert out[0] and out[1]
