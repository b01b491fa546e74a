"""blocksparse_attn_fwd_noalloc: the attention call for callers that cannot
allocate device memory (plug-in hosts without an allocator, loops where a
cudaMalloc is not acceptable).  It keeps its scratch in the library's static
device array instead of a caller workspace.  Checked through the C ABI
against the workspace entry point on two calls in a row with different
shapes, so the second call runs over what the first left in the array.

This file is collected last on purpose, so that a run stopping at its first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_lvsa_b200 import inputs
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


def one_call(bsa, wl, s):
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    o_ref, lse_ref = bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale)
    o = torch.empty_like(q)
    lse = torch.empty((wl.H, wl.N), dtype=torch.float32, device="cuda")
    bsa.blocksparse_attn_fwd_noalloc(q, k, v, ix, o, lse, scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    err = (o.double() - o_ref.double()).abs()
    assert err.max().item() <= gu.O_MAX and err.mean().item() <= gu.O_MEAN
    assert (lse.double() - lse_ref.double()).abs().max().item() <= gu.LSE_MAX


def test_noalloc_matches_workspace_call_twice(bsa):
    # first call: 1x horizon (256 query tiles); second call: 6x horizon (1536 tiles)
    one_call(bsa, WORKLOADS["wan1.3b_1x_c11"], 0)
    one_call(bsa, WORKLOADS["wan1.3b_6x"], 1)


def test_noalloc_rejects_oversize_before_launch(bsa):
    # 2000 query tiles need ~20 MB of tile lists: more than the static array holds
    ix = bsa.bsa_index()
    ix.kind = bsa.BSA_INDEX_LVSA_FRAMES
    ix.T = 100
    ix.frames = ix.counts = 0x10000          # never read: rejected on the host
    fake = ctypes.c_void_p(0x10000)
    rc = bsa.lib().blocksparse_attn_fwd_noalloc(fake, fake, fake, 256000, 1, 128, 0.1, ctypes.byref(ix),
                                                fake, fake, ctypes.c_void_p(0))
    assert rc == bsa.BSA_ERR_WORKSPACE
