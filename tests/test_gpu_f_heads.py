"""GPU parity of the head-sharded use (one GPU stands in for one rank): the C
ABI called on a rank's contiguous head range, sliced out of the full
[N, H, d] tensors, gives for those heads exactly what the call on all heads
gives (bit for bit: heads are independent in the kernels), and matches the
oracle on sampled rows.  Uneven ranges: 12 heads over 5 ranks (3, 3, 2, 2, 2)
and 40 heads over 3 ranks (14, 13, 13)."""
import numpy as np
import pytest
import torch

from oracle import losa as olosa
from oracle import lvsa as olvsa
from block_sparse_attention_lvsa_b200 import heads, inputs
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


@pytest.mark.parametrize("world,rank", [(5, 1), (5, 4)])
def test_lvsa_head_shard(bsa, world, rank):
    wl = WORKLOADS["wan1.3b_1x_c11"]
    s = 3
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    o_all, lse_all = bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale)
    h0, h1 = heads.head_range(wl.H, world, rank)
    ql, kl, vl = (heads.local_heads(x, wl.H, world, rank) for x in (q, k, v))
    o, lse = bsa.blocksparse_attn_fwd(ql, kl, vl, ix, scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o, o_all[:, h0:h1]) and torch.equal(lse, lse_all[h0:h1])
    # the oracle on the global heads, compared with the local outputs
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, s)
    rows = inputs.sample_rows(wl.N, wl.P, 96, 80 + rank).numpy()
    keys, group = gu.lvsa_keys(A, wl.P, wl.N)
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, [h0, h1 - 1], keys, group)
    local = {h - h0: Os[h] for h in Os}, {h - h0: Ls[h] for h in Ls}
    gu.compare_rows(o, lse, local[0], local[1], rows, f"lvsa shard {rank}/{world}")


@pytest.mark.parametrize("world,rank", [(3, 1), (3, 2)])
def test_losa_head_shard(bsa, world, rank):
    wl = WORKLOADS["wan14b_losa"]
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    o_all, lse_all, mass_all = bsa.attn_dense_blockmass(q, k, v, 128, wl.scale)
    h0, h1 = heads.head_range(wl.H, world, rank)
    ql, kl, vl = (heads.local_heads(x, wl.H, world, rank) for x in (q, k, v))
    o, lse, mass = bsa.attn_dense_blockmass(ql, kl, vl, 128, wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o, o_all[:, h0:h1]) and torch.equal(lse, lse_all[h0:h1])
    assert torch.equal(mass, mass_all[h0:h1])
    # selection on the shard's mass: bit-exact against the oracle
    idx, cnt = bsa.losa_select(mass, wl.tau)
    assert bsa.get_device_status() == bsa.BSA_OK
    ref_idx, ref_cnt = olosa.select(mass.cpu().numpy(), wl.tau)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    # a later step with the shard's frozen index, against the oracle on the global heads
    q1, k1, v1 = inputs.workload_qkv(wl, 5, device="cuda")
    ql1, kl1, vl1 = (heads.local_heads(x, wl.H, world, rank) for x in (q1, k1, v1))
    o1, lse1 = bsa.blocksparse_attn_fwd(ql1, kl1, vl1, bsa.block_index(idx, cnt), scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    rows = inputs.sample_rows(wl.N, wl.P, 96, 90 + rank).numpy()
    idx_np, cnt_np = idx.cpu().numpy(), cnt.cpu().numpy()
    keys_l, group = gu.block_keys(idx_np, cnt_np, wl.N)
    hs = [h0, h1 - 1]
    Os, Ls = gu.oracle_rows(q1, k1, v1, wl.scale, rows, hs, lambda h, r: keys_l(h - h0, r), group)
    gu.compare_rows(o1, lse1, {h - h0: Os[h] for h in hs}, {h - h0: Ls[h] for h in hs}, rows,
                    f"losa shard {rank}/{world}")
