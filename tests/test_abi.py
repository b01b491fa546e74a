"""The C-ABI library builds, loads and exports every declared symbol; host-side
argument validation (no GPU work is enqueued by any call in this file)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import build
    build.build()
    from block_sparse_attention_lvsa_b200 import binding
    return binding


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**([a-z_][a-z0-9_]*)\s*\(",
                       src, flags=re.M)
    return sorted(set(names))


def test_header_declares_the_four_calls():
    names = declared_functions()
    for n in ("lvsa_build_index", "attn_dense_blockmass", "losa_select", "blocksparse_attn_fwd"):
        assert n in names


def test_every_declared_symbol_exported(bsa):
    lib = ctypes.CDLL(bsa.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) <= set(bsa.EXPORTED)


def test_status_strings(bsa):
    assert bsa.status_string(0) == "BSA_OK"
    assert bsa.status_string(-5) == "BSA_ERR_TIMEOUT"
    assert bsa.status_string(12345) == "BSA_UNKNOWN_STATUS"


def test_workspace_bytes(bsa):
    ix = bsa.bsa_index()
    ix.kind = bsa.BSA_INDEX_LVSA_FRAMES
    ix.T = 126
    n = bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, 196560, 12, 128, ix)
    nB = 1536
    assert n >= nB * nB * 5 and n % 256 == 0
    ix.kind = bsa.BSA_INDEX_BLOCKS
    assert bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, 32760, 40, 128, ix) == 0
    share = 256 * 32760 * 4                        # key tiles x rows x float32, one head
    assert bsa.workspace_bytes(bsa.BSA_OP_DENSE_BLOCKMASS, 32760, 40, 128, None) == 40 * share
    share720 = 1772 * 226800 * 4                   # 720p: two heads fit in 4 GiB
    assert bsa.workspace_bytes(bsa.BSA_OP_DENSE_BLOCKMASS, 226800, 40, 128, None) == 2 * share720
    assert bsa.workspace_bytes(bsa.BSA_OP_DENSE_BLOCKMASS, 4 * 10 ** 6, 1, 128, None) == 31250 * 4 * 10 ** 6 * 4
    with pytest.raises(bsa.BsaError):
        bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, 100, 1, 128, None)
    ix.kind = bsa.BSA_INDEX_LVSA_FRAMES
    ix.T = 7
    with pytest.raises(bsa.BsaError):      # T does not divide N
        bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, 100, 1, 128, ix)
    # intersection: the LVSA lists plus one flag byte per (head, query block, key block)
    ix.kind, ix.T = bsa.BSA_INDEX_LVSA_FRAMES, 126
    lv = bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, 196560, 12, 128, ix)
    ix.kind = bsa.BSA_INDEX_LVSA_BLOCKS
    both = bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, 196560, 12, 128, ix)
    assert both == lv + 12 * 1536 * 1536
    # restricted mass: index part (256-aligned) + one share of log partial sums per head, all 12 here
    share = 1536 * 196560 * 4
    assert bsa.workspace_bytes(bsa.BSA_OP_BLOCKMASS, 196560, 12, 128, ix) == both + 1 * share or \
        bsa.workspace_bytes(bsa.BSA_OP_BLOCKMASS, 196560, 12, 128, ix) == both + (4 << 30) // share * share
    ix.kind = bsa.BSA_INDEX_BLOCKS
    assert bsa.workspace_bytes(bsa.BSA_OP_BLOCKMASS, 32760, 40, 128, ix) == 40 * 256 * 32760 * 4


def test_host_validation_rejects_before_launch(bsa):
    L = bsa.lib()
    nul = ctypes.c_void_p(0)
    fake = ctypes.c_void_p(0x10000)     # never dereferenced: rejected on the host first
    assert L.lvsa_build_index(0, 4, 3, 4, 0, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index(8, 0, 3, 4, 0, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index(8, 4, 3, 4, -1, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index(8, 4, 3, 4, 0, nul, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index(2000, 4, 3, 4, 0, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index_window(0, 4, 3, 0, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index_window(8, 4, 0, 0, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index_window(8, 4, 3, -1, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert L.lvsa_build_index_window(8, 4, 3, 0, fake, nul, nul) == bsa.BSA_ERR_ARG
    ix = bsa.bsa_index()
    ix.kind = bsa.BSA_INDEX_LVSA_FRAMES
    ix.T = 8
    ix.frames = ix.counts = 0x10000
    f = L.blocksparse_attn_fwd
    # unsupported head size
    assert f(fake, fake, fake, 512, 2, 96, 0.1, ctypes.byref(ix), fake, fake, fake, 1 << 30, nul) == bsa.BSA_ERR_UNSUPPORTED
    # null output
    assert f(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(ix), nul, fake, fake, 1 << 30, nul) == bsa.BSA_ERR_ARG
    # misaligned q
    assert f(ctypes.c_void_p(0x10002), fake, fake, 512, 2, 64, 0.1, ctypes.byref(ix), fake, fake, fake, 1 << 30, nul) == bsa.BSA_ERR_ARG
    # T does not divide N
    assert f(fake, fake, fake, 500, 2, 64, 0.1, ctypes.byref(ix), fake, fake, fake, 1 << 30, nul) == bsa.BSA_ERR_SHAPE
    # workspace too small
    assert f(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(ix), fake, fake, fake, 16, nul) == bsa.BSA_ERR_WORKSPACE
    # non-finite scale
    assert f(fake, fake, fake, 512, 2, 64, float("nan"), ctypes.byref(ix), fake, fake, fake, 1 << 30, nul) == bsa.BSA_ERR_ARG
    ix.kind = bsa.BSA_INDEX_BLOCKS
    ix.block, ix.H, ix.nQB, ix.nKB = 64, 2, 4, 4
    ix.idx = ix.cnt = 0x10000
    assert f(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(ix), fake, fake, nul, 0, nul) == bsa.BSA_ERR_UNSUPPORTED
    ix.block = 128
    ix.nKB = 5
    assert f(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(ix), fake, fake, nul, 0, nul) == bsa.BSA_ERR_SHAPE
    ix.kind = 9
    assert f(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(ix), fake, fake, nul, 0, nul) == bsa.BSA_ERR_ARG
    g = L.attn_dense_blockmass
    assert g(fake, fake, fake, 512, 2, 64, 64, 0.1, fake, fake, fake, nul, 0, nul) == bsa.BSA_ERR_UNSUPPORTED
    assert g(fake, fake, fake, 512, 2, 64, 128, 0.1, fake, fake, nul, nul, 0, nul) == bsa.BSA_ERR_ARG
    # the one-pass mass needs at least one head's share of workspace: 4 key tiles x 512 rows x 4 bytes
    assert g(fake, fake, fake, 512, 2, 64, 128, 0.1, fake, fake, fake, nul, 0, nul) == bsa.BSA_ERR_WORKSPACE
    assert g(fake, fake, fake, 512, 2, 64, 128, 0.1, fake, fake, fake, fake, 4 * 512 * 4 - 1, nul) == bsa.BSA_ERR_WORKSPACE
    m = L.attn_blockmass
    assert m(fake, fake, fake, 512, 2, 64, 0.1, None, fake, fake, fake, fake, 1 << 20, nul) == bsa.BSA_ERR_ARG
    bix = bsa.bsa_index()
    bix.kind = bsa.BSA_INDEX_LVSA_BLOCKS
    bix.T, bix.frames, bix.counts = 8, 0x10000, 0x10000
    bix.block, bix.H, bix.nQB, bix.nKB, bix.idx, bix.cnt = 128, 3, 4, 4, 0x10000, 0x10000
    assert m(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(bix), fake, fake, fake, fake, 1 << 20, nul) == \
        bsa.BSA_ERR_SHAPE                                   # H of the block lists != H
    bix.H = 2
    assert m(fake, fake, fake, 512, 2, 64, 0.1, ctypes.byref(bix), fake, fake, fake, fake, 100, nul) == \
        bsa.BSA_ERR_WORKSPACE                               # too small for the lists, before any launch
    s = L.losa_select
    assert s(fake, 2, 4, 4, 0.0, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert s(fake, 2, 4, 4, 1.5, fake, fake, nul) == bsa.BSA_ERR_ARG
    assert s(fake, 2, 4, 9000, 0.99, fake, fake, nul) == bsa.BSA_ERR_UNSUPPORTED
    assert L.bsa_debug_expired_wait(10, 0, nul) == bsa.BSA_ERR_ARG
    assert L.bsa_debug_expired_wait(1_000_000, 2, nul) == bsa.BSA_ERR_ARG


def test_output_checks_reject_wrong_buffers(bsa):
    """Caller-supplied outputs and index arrays are checked before any call:
    the library sees only pointers, so an undersized or mistyped buffer would
    mean out-of-bounds device writes (CPU tensors stand in for device ones)."""
    import torch
    N, H, d = 300, 2, 64
    q = torch.zeros((N, H, d), dtype=torch.bfloat16)
    ok_o = torch.zeros_like(q)
    ok_lse = torch.zeros((H, N), dtype=torch.float32)
    bsa._check_out(q, ok_o, ok_lse)                                     # accepted
    bad = [
        (torch.zeros((N, H, d), dtype=torch.float32), ok_lse),          # o dtype
        (torch.zeros((N - 1, H, d), dtype=torch.bfloat16), ok_lse),     # o shape
        (torch.zeros((N, H, 2 * d), dtype=torch.bfloat16)[:, :, ::2], ok_lse),   # o not contiguous
        (ok_o, torch.zeros((N, H), dtype=torch.float32)),               # lse transposed
        (ok_o, torch.zeros((H, N), dtype=torch.float64)),               # lse dtype
        (ok_o.to("meta"), ok_lse),                                      # o on another device
    ]
    for o, lse in bad:
        with pytest.raises(ValueError):
            bsa._check_out(q, o, lse)
    nB = 3
    with pytest.raises(ValueError):
        bsa._check_out(q, ok_o, ok_lse, torch.zeros((H, nB, nB - 1), dtype=torch.float32))
    with pytest.raises(ValueError):                                     # int64 block index
        bsa.block_index(torch.zeros((H, nB, nB), dtype=torch.int64), torch.zeros((H, nB), dtype=torch.int32))
    with pytest.raises(ValueError):                                     # cnt of the wrong shape
        bsa.block_index(torch.zeros((H, nB, nB), dtype=torch.int32), torch.zeros((H, nB + 1), dtype=torch.int32))
    with pytest.raises(ValueError):                                     # frames not [T, T]
        bsa.lvsa_index(5, torch.zeros((5, 4), dtype=torch.int32), torch.zeros(5, dtype=torch.int32))
    with pytest.raises(ValueError):                                     # no-alloc needs o and lse
        bsa.blocksparse_attn_fwd_noalloc(q, q, q, bsa.bsa_index(), None, None)
