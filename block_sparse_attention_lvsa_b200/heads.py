"""Head-sharded use of the kernels across GPUs: one process per GPU.

Attention heads are independent in both methods: the LVSA frame sets
A(t) are the same for every head ("LVSA: Training-Free Sparse Attention for
Long Video Diffusion", technical summary section 2), and the LoSA block
mass, selection and frozen index are per head ("LoSA (Near-Lossless Sparse
Attention)", section "Balancing efficiency and quality").  So a rank that
holds q, k, v of a contiguous head range [h0, h1) runs every call of the
library on those heads alone, with no exchange inside the path.  When a
caller needs the whole result on every rank, ``gather_heads`` assembles
O [N, H, d] and LSE [H, N] with one all-gather per tensor
(torch.distributed: NCCL over NVLink between GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch


def head_range(H: int, world: int, rank: int) -> Tuple[int, int]:
    """Heads [h0, h1) of `rank` among `world` ranks: contiguous, sizes differ
    by at most one, the first H % world ranks holding the larger share."""
    if H < 1 or world < 1 or not 0 <= rank < world:
        raise ValueError("need H >= 1, world >= 1, 0 <= rank < world")
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def local_heads(x: torch.Tensor, H: int, world: int, rank: int, head_dim: int = 1) -> torch.Tensor:
    """The rank's slice of a tensor with heads on `head_dim` (q, k, v [N, H, d]
    use 1; LSE [H, N] and LoSA mass [H, nB, nB] use 0), made contiguous."""
    h0, h1 = head_range(H, world, rank)
    return x.narrow(head_dim, h0, h1 - h0).contiguous()


def gather_heads(o_local: torch.Tensor, lse_local: torch.Tensor, H: int,
                 group: Optional[object] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """All ranks' O [N, h1-h0, d] and LSE [h1-h0, N] assembled into O [N, H, d]
    and LSE [H, N] on every rank.  Shards are padded to the largest share so
    one fixed-size all-gather per tensor serves uneven head counts."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    h0, h1 = head_range(H, world, rank)
    if o_local.shape[1] != h1 - h0 or lse_local.shape[0] != h1 - h0:
        raise ValueError("local shards do not match this rank's head range")
    width = -(-H // world)
    N, _, d = o_local.shape
    o_pad = o_local.new_zeros((N, width, d))
    o_pad[:, :h1 - h0] = o_local
    l_pad = lse_local.new_zeros((width, N))
    l_pad[:h1 - h0] = lse_local
    # 2-byte floats travel bit for bit as pairs in int32 (even d), else as
    # float32 (exact both ways): every backend moves those types
    two_byte = o_pad.element_size() == 2 and o_pad.is_floating_point()
    if two_byte and d % 2 == 0:
        o_send = o_pad.view(torch.int32)
    elif two_byte:
        o_send = o_pad.float()
    else:
        o_send = o_pad
    o_parts = [torch.empty_like(o_send) for _ in range(world)]
    l_parts = [torch.empty_like(l_pad) for _ in range(world)]
    dist.all_gather(o_parts, o_send, group=group)
    dist.all_gather(l_parts, l_pad, group=group)
    if two_byte and d % 2 == 0:
        o_parts = [t.view(o_pad.dtype) for t in o_parts]
    elif two_byte:
        o_parts = [t.to(o_pad.dtype) for t in o_parts]
    o_full = o_local.new_empty((N, H, d))
    l_full = lse_local.new_empty((H, N))
    for r in range(world):
        a, b = head_range(H, world, r)
        o_full[:, a:b] = o_parts[r][:, :b - a]
        l_full[a:b] = l_parts[r][:b - a]
    return o_full, l_full
