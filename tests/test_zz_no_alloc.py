"""blocksparse_attn_fwd_noalloc: the attention call for callers that cannot
allocate device memory (plug-in hosts that own every device buffer and give a
plug-in no allocator, loops where a cudaMalloc is not acceptable).  It keeps
its scratch in the library's static device array instead of a caller
workspace.  Both entry points run the same kernels on the same inputs, so
their outputs must be identical bit for bit; they are checked against each
other through the C ABI on two calls in a row with different shapes (the
second call runs over what the first left in the array), and sampled rows
are checked against the oracle.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test."""
import ctypes

import pytest
import torch

from oracle import lvsa as olvsa
from block_sparse_attention_lvsa_b200 import inputs
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


def one_call(bsa, wl, s, rows_n, heads, seed):
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    o_ref, lse_ref = bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale)
    o = torch.empty_like(q)
    lse = torch.empty((wl.H, wl.N), dtype=torch.float32, device="cuda")
    bsa.blocksparse_attn_fwd_noalloc(q, k, v, ix, o, lse, scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, s)
    rows = inputs.sample_rows(wl.N, wl.P, rows_n, seed).numpy()
    keys, group = gu.lvsa_keys(A, wl.P, wl.N)
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, heads, keys, group)
    gu.compare_rows(o, lse, Os, Ls, rows, f"noalloc {wl.name} s={s}")


def test_noalloc_matches_workspace_call_twice(bsa):
    # first call: 1x horizon (256 query tiles); second call: 6x horizon (1536 tiles)
    one_call(bsa, WORKLOADS["wan1.3b_1x_c11"], 0, 96, [0, 7], 70)
    one_call(bsa, WORKLOADS["wan1.3b_6x"], 1, 96, [3], 71)


def test_noalloc_intersection_index(bsa):
    """The intersection kind fits the static array at the 1x-horizon shape."""
    wl = WORKLOADS["wan1.3b_1x_c11"]
    q, k, v = inputs.workload_qkv(wl, 2, device="cuda")
    nB = -(-wl.N // 128)
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 2, device="cuda")
    g = torch.Generator().manual_seed(5)
    keep = torch.rand((wl.H, nB, nB), generator=g) < 0.5
    keep[:, torch.arange(nB), torch.arange(nB)] = True
    cnt = keep.sum(dim=2).to(torch.int32)
    order = torch.sort((~keep).to(torch.int32) * nB + torch.arange(nB), dim=2).values
    idx = torch.where(order < nB, order, torch.full_like(order, -1)).to(torch.int32)
    idx_d, cnt_d = idx.cuda(), cnt.cuda()
    ix3 = bsa.lvsa_block_index(wl.T, frames, counts, idx_d, cnt_d)
    o_ref, lse_ref = bsa.blocksparse_attn_fwd(q, k, v, ix3, scale=wl.scale)
    o, lse = torch.empty_like(q), torch.empty((wl.H, wl.N), dtype=torch.float32, device="cuda")
    bsa.blocksparse_attn_fwd_noalloc(q, k, v, ix3, o, lse, scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o, o_ref)
    assert torch.equal(lse, lse_ref)


def test_noalloc_rejects_oversize_before_launch(bsa):
    fake = ctypes.c_void_p(0x10000)          # never read: rejected on the host
    # frame lists: 2000 query tiles need ~20 MB of tile lists
    ix = bsa.bsa_index()
    ix.kind = bsa.BSA_INDEX_LVSA_FRAMES
    ix.T = 100
    ix.frames = ix.counts = 0x10000
    rc = bsa.lib().blocksparse_attn_fwd_noalloc(fake, fake, fake, 256000, 1, 128, 0.1, ctypes.byref(ix),
                                                fake, fake, ctypes.c_void_p(0))
    assert rc == bsa.BSA_ERR_WORKSPACE
    # intersection at the 720p 14B-head shape: 40 * 1772^2 flag bytes alone are ~125 MB
    ix3 = bsa.bsa_index()
    ix3.kind = bsa.BSA_INDEX_LVSA_BLOCKS
    ix3.T = 63
    ix3.frames = ix3.counts = ix3.idx = ix3.cnt = 0x10000
    ix3.block, ix3.H, ix3.nQB, ix3.nKB = 128, 40, 1772, 1772
    rc = bsa.lib().blocksparse_attn_fwd_noalloc(fake, fake, fake, 226800, 40, 128, 0.1, ctypes.byref(ix3),
                                                fake, fake, ctypes.c_void_p(0))
    assert rc == bsa.BSA_ERR_WORKSPACE
