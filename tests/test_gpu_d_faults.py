"""Kernel-side failure reporting without faulting the GPU: an expired bounded
wait and out-of-range frame ids are reported through the status word, and the
context stays usable afterwards."""
import numpy as np
import pytest
import torch

from block_sparse_attention_lvsa_b200 import inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


def small_call(bsa):
    q, k, v = inputs.make_qkv(512, 2, 64, seed=1, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(8, 4, 3, 4, 0, device="cuda")
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(8, frames, counts))
    return o


@pytest.mark.parametrize("form", [0, 1])
def test_expired_wait_reports_timeout(bsa, form):
    """form 0: one thread waits; 1: the whole warp waits (the MMA issuer's form)."""
    assert bsa.get_device_status() == bsa.BSA_OK
    assert bsa.debug_expired_wait(20_000_000, form) == bsa.BSA_OK   # 20 ms
    assert bsa.get_device_status() == bsa.BSA_ERR_TIMEOUT
    o = small_call(bsa)                                              # context still usable
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.isfinite(o.float()).all()


def test_frame_out_of_range_reported(bsa):
    q, k, v = inputs.make_qkv(512, 2, 64, seed=2, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(8, 4, 3, 4, 0, device="cuda")
    frames[3, 1] = 99
    bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(8, frames, counts))
    assert bsa.get_device_status() == bsa.BSA_ERR_INDEX_RANGE
    counts[2] = 50
    bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(8, frames, counts))
    assert bsa.get_device_status() == bsa.BSA_ERR_INDEX_RANGE
    small_call(bsa)
    assert bsa.get_device_status() == bsa.BSA_OK


def test_block_count_out_of_range_reported(bsa):
    N, H, d = 512, 2, 64
    q, k, v = inputs.make_qkv(N, H, d, seed=3, device="cuda")
    idx = torch.arange(4, dtype=torch.int32, device="cuda").repeat(H, 4, 1)
    cnt = torch.full((H, 4), 4, dtype=torch.int32, device="cuda")
    cnt[1, 2] = 9
    bsa.blocksparse_attn_fwd(q, k, v, bsa.block_index(idx, cnt))
    assert bsa.get_device_status() == bsa.BSA_ERR_INDEX_RANGE
