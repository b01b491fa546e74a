"""GPU: the calls bench.py times from a CUDA graph (the microsecond-scale
ones) record their launches on the capturing stream, and a replay gives the
same outputs, bit for bit, as the eager call.

A call that launched on some other stream would leave the graph empty and
its replay would time nothing; torch reports that as a warning, which these
tests turn into an error.
"""
import warnings

import pytest
import torch

from block_sparse_attention_lvsa_b200 import inputs
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


def capture(fn):
    """fn() captured once into a CUDA graph on a side stream (current stream
    during capture); an empty capture is an error."""
    fn()                                    # first call outside capture
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with warnings.catch_warnings():
        warnings.filterwarnings("error", message=".*CUDA Graph is empty.*")
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                fn()
    return g


def test_attention_call_replays_bit_identical(bsa):
    wl = WORKLOADS["tiny"]
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 1, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    q, k, v = inputs.workload_qkv(wl, 1, device="cuda")
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, wl.N, wl.H, wl.d, ix), dtype=torch.uint8,
                     device="cuda")
    o_ref, lse_ref = bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale, workspace=ws)
    torch.cuda.synchronize()
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(lse_ref)
    g = capture(lambda: bsa.blocksparse_attn_fwd(q, k, v, ix, scale=wl.scale, o=o, lse=lse, workspace=ws))
    o.zero_()
    lse.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o, o_ref) and torch.equal(lse, lse_ref)


def test_index_build_replays_bit_identical(bsa):
    wl = WORKLOADS["wan1.3b_6x"]
    f_ref, c_ref, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 3, device="cuda")
    frames = torch.empty_like(f_ref)
    counts = torch.empty_like(c_ref)
    g = capture(lambda: bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, 3, frames, counts))
    frames.fill_(-7)
    counts.fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(frames, f_ref) and torch.equal(counts, c_ref)


def test_selection_replays_bit_identical(bsa):
    gen = torch.Generator(device="cuda").manual_seed(5)
    w = torch.exp(torch.randn((3 * 40, 300), generator=gen, device="cuda") * 2.5)
    mass = (w / w.sum(dim=1, keepdim=True) * 128).float().view(3, 40, 300).contiguous()
    i_ref, c_ref = bsa.losa_select(mass, 0.99)
    torch.cuda.synchronize()
    idx = torch.empty_like(i_ref)
    cnt = torch.empty_like(c_ref)
    g = capture(lambda: bsa.losa_select(mass, 0.99, idx=idx, cnt=cnt))
    idx.fill_(-7)
    cnt.fill_(-7)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(idx, i_ref) and torch.equal(cnt, c_ref)
