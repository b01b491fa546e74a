"""GPU parity: dense attention + block mass, LoSA selection, frozen-index reuse."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import losa as olosa
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
from block_sparse_attention_lvsa_b200 import inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


def rows_in_block(N, nB):
    return np.array([min((b + 1) * 128, N) - b * 128 for b in range(nB)], dtype=np.float64)


@pytest.mark.parametrize("N,H,d", [(600, 2, 64), (600, 2, 128), (256, 1, 128), (77, 3, 64), (1000, 2, 128)])
def test_dense_blockmass_small(bsa, N, H, d):
    q, k, v = inputs.make_qkv(N, H, d, seed=N + d, device="cuda")
    scale = d ** -0.5
    o, lse, mass = bsa.attn_dense_blockmass(q, k, v, 128, scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    qn, kn, vn = (x.cpu().double().numpy() for x in (q, k, v))
    O, L = oatt.attention_dense_masked(qn, kn, vn, scale, np.ones((N, N), dtype=bool))
    err = np.abs(o.cpu().double().numpy() - O)
    assert err.max() <= gu.O_MAX and err.mean() <= gu.O_MEAN
    assert np.abs(lse.cpu().double().numpy() - L).max() <= gu.LSE_MAX
    nB = -(-N // 128)
    ref = oatt.block_mass(qn, kn, scale, 128, range(H), range(nB))
    mg = mass.cpu().double().numpy()
    sizes = rows_in_block(N, nB)
    for h in range(H):
        for qb in range(nB):
            e = np.abs(mg[h, qb] - ref[(h, qb)]).max() / sizes[qb]
            assert e <= gu.MASS_MAX, (h, qb, e)


@pytest.mark.parametrize("N,H,d", [(1000, 3, 128), (300, 5, 64)])
def test_dense_blockmass_head_passes(bsa, N, H, d):
    """A workspace of one head's share (one pass per head) and of two shares
    give the same o, lse and mass bit for bit as all heads in one pass."""
    q, k, v = inputs.make_qkv(N, H, d, seed=7 * N + d, device="cuda")
    share = (-(-N // 128)) * N * 4
    full = bsa.attn_dense_blockmass(q, k, v, 128, d ** -0.5)
    assert bsa.get_device_status() == bsa.BSA_OK
    for shares in (1, 2):
        ws = torch.empty(shares * share + 100, dtype=torch.uint8, device="cuda")
        part = bsa.attn_dense_blockmass(q, k, v, 128, d ** -0.5, workspace=ws)
        assert bsa.get_device_status() == bsa.BSA_OK
        for a, b in zip(full, part):
            assert torch.equal(a, b)
    with pytest.raises(bsa.BsaError):
        bsa.attn_dense_blockmass(q, k, v, 128, d ** -0.5,
                                 workspace=torch.empty(share - 4, dtype=torch.uint8, device="cuda"))


@pytest.fixture(scope="module")
def losa_step0(bsa):
    """Dense measuring step on the 14B-shaped LoSA workload (full size)."""
    wl = WORKLOADS["wan14b_losa"]
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    o, lse, mass = bsa.attn_dense_blockmass(q, k, v, wl.block, wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    return wl, (q, k, v), o, lse, mass


def test_losa_mass_full_size(bsa, losa_step0):
    wl, (q, k, v), o, lse, mass = losa_step0
    nB = mass.shape[1]
    # every (head, query block): masses sum to the number of rows of the block
    sums = mass.double().sum(dim=2).cpu().numpy()
    sizes = rows_in_block(wl.N, nB)
    assert np.abs(sums / sizes[None, :] - 1.0).max() < 1e-4
    # sampled (head, query block) rows against the oracle's dense probabilities
    rng = np.random.default_rng(4)
    mg = mass.cpu().double().numpy()
    for h in (0, 17, 39):
        qh, kh = gu.head_f64(q, h), gu.head_f64(k, h)
        qbs = sorted(set([0, nB - 1] + rng.integers(0, nB, 6).tolist()))
        ref = oatt.block_mass(qh, kh, wl.scale, 128, [0], qbs)
        for qb in qbs:
            e = np.abs(mg[h, qb] - ref[(0, qb)]).max() / sizes[qb]
            assert e <= gu.MASS_MAX, (h, qb, e)
    # dense output, sampled rows
    rows = inputs.sample_rows(wl.N, wl.P, 96, 8).numpy()
    keys, group = gu.dense_keys(wl.N)
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, [1, 38], keys, group)
    gu.compare_rows(o, lse, Os, Ls, rows, "losa dense step")


def test_losa_select_bitexact_on_gpu_mass(bsa, losa_step0):
    wl, _, _, _, mass = losa_step0
    idx, cnt = bsa.losa_select(mass, wl.tau)
    assert bsa.get_device_status() == bsa.BSA_OK
    ref_idx, ref_cnt = olosa.select(mass.cpu().numpy(), wl.tau)
    assert np.array_equal(cnt.cpu().numpy(), ref_cnt)
    assert np.array_equal(idx.cpu().numpy(), ref_idx)
    kept = float(ref_cnt.sum()) / ref_cnt.size / mass.shape[2]
    assert 0.0 < kept < 1.0


@pytest.mark.parametrize("nKB", [1, 2, 7, 128, 256, 257, 700, 1772, 3000, 8192])
def test_losa_select_random(bsa, nKB):
    rng = np.random.default_rng(nKB)
    H, nQB = 2, 3
    m = rng.random((H, nQB, nKB)) ** 6
    m[0, 0] = 0.25                               # all ties
    m[1, 1, ::3] = 0.0                           # zeros
    m = (m * 128.0 / np.maximum(m.sum(axis=2, keepdims=True), 1e-30)).astype(np.float32)
    m[0, 1] = 0.0                                # all-zero row
    mass = torch.from_numpy(m).cuda()
    for tau in (0.99, 0.5, 1.0, 1e-9):
        idx, cnt = bsa.losa_select(mass, tau)
        assert bsa.get_device_status() == bsa.BSA_OK
        ref_idx, ref_cnt = olosa.select(m, tau)
        assert np.array_equal(cnt.cpu().numpy(), ref_cnt), tau
        assert np.array_equal(idx.cpu().numpy(), ref_idx), tau


@pytest.mark.parametrize("nKB", [5, 256, 1772])
def test_losa_select_q_collisions(bsa, nKB):
    """Distinct masses below 2^-9 share Q = floor(mass * 2^33): the (Q desc, kb asc)
    order must decide among them by kb, not by mass; -0.0 counts as zero."""
    rng = np.random.default_rng(100 + nKB)
    H, nQB = 2, 4
    m = ((rng.integers(0, 4, (H, nQB, nKB)) + rng.random((H, nQB, nKB))) * 2.0 ** -33).astype(np.float32)
    m[0, 1, :: 4] = 2.0 ** -20                                 # a few larger, tied masses
    m[1, 2, 0] = 64.0                                          # one dominant block
    m[1, 3, 1::2] = -0.0
    mass = torch.from_numpy(m).cuda()
    for tau in (0.99, 0.5, 1.0):
        idx, cnt = bsa.losa_select(mass, tau)
        assert bsa.get_device_status() == bsa.BSA_OK
        ref_idx, ref_cnt = olosa.select(m, tau)
        assert np.array_equal(cnt.cpu().numpy(), ref_cnt), tau
        assert np.array_equal(idx.cpu().numpy(), ref_idx), tau


@pytest.mark.parametrize("n_zero", [0, 43, 2000])
def test_losa_select_large_total(bsa, n_zero):
    """Row totals above 2^53 whose float64 conversion rounds up (the threshold is
    clamped to the total): the register kernel (<= 2048 blocks) and the
    shared-memory kernel (longer rows) must both keep exactly the oracle's set."""
    from tests.test_oracle_losa import large_total_row
    row = large_total_row(n_zero)
    m = np.stack([row, row[::-1].copy()])[None]              # [1, 2, nKB]
    mass = torch.from_numpy(np.ascontiguousarray(m)).cuda()
    for tau in (1.0, 0.99):
        idx, cnt = bsa.losa_select(mass, tau)
        assert bsa.get_device_status() == bsa.BSA_OK
        ref_idx, ref_cnt = olosa.select(m, tau)
        assert np.array_equal(cnt.cpu().numpy(), ref_cnt), tau
        assert np.array_equal(idx.cpu().numpy(), ref_idx), tau


def test_losa_select_rejects_bad_mass(bsa):
    m = torch.tensor([[[0.5, float("nan"), -1.0, 3.0]]], dtype=torch.float32, device="cuda")
    bsa.losa_select(m, 0.99)
    assert bsa.get_device_status() == bsa.BSA_ERR_ARG
    assert bsa.get_device_status() == bsa.BSA_OK        # cleared by the read


@pytest.mark.parametrize("s", [1, 20, 39])
def test_frozen_reuse(bsa, losa_step0, s):
    wl, _, _, _, mass = losa_step0
    idx, cnt = bsa.losa_select(mass, wl.tau)
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.block_index(idx, cnt), scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    rows = inputs.sample_rows(wl.N, wl.P, 96, 60 + s).numpy()
    keys, group = gu.block_keys(idx.cpu().numpy(), cnt.cpu().numpy(), wl.N)
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, [2, 33], keys, group)
    gu.compare_rows(o, lse, Os, Ls, rows, f"losa reuse s={s}")


def test_block_index_edge_cases(bsa):
    N, H, d = 700, 2, 128
    nB = -(-N // 128)
    q, k, v = inputs.make_qkv(N, H, d, seed=11, device="cuda")
    rng = np.random.default_rng(6)
    idx = np.full((H, nB, nB), -1, dtype=np.int32)
    cnt = np.zeros((H, nB), dtype=np.int32)
    for h in range(H):
        for qb in range(nB):
            if (h, qb) == (0, 2):
                continue                           # empty row: O = 0, LSE = -inf
            kept = sorted(rng.choice(nB, size=int(rng.integers(1, nB + 1)), replace=False).tolist())
            idx[h, qb, :len(kept)] = kept
            cnt[h, qb] = len(kept)
    it, ct = torch.from_numpy(idx).cuda(), torch.from_numpy(cnt).cuda()
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.block_index(it, ct))
    assert bsa.get_device_status() == bsa.BSA_OK
    rows = np.arange(N)
    keys, group = gu.block_keys(idx, cnt, N)
    Os, Ls = gu.oracle_rows(q, k, v, d ** -0.5, rows, range(H), keys, group)
    gu.compare_rows(o, lse, Os, Ls, rows, "block edge cases")
    assert torch.all(o[256:384, 0] == 0) and torch.all(torch.isneginf(lse[0, 256:384]))
    # an out-of-range entry is skipped and reported
    idx2 = idx.copy()
    idx2[1, 0, 0] = nB + 5
    o2, lse2 = bsa.blocksparse_attn_fwd(q, k, v, bsa.block_index(torch.from_numpy(idx2).cuda(), ct))
    assert bsa.get_device_status() == bsa.BSA_ERR_INDEX_RANGE
    cnt3 = cnt.copy()
    idx3 = idx.copy()
    kept = [kb for kb in idx[1, 0, :cnt[1, 0]] if kb != idx[1, 0, 0]]
    idx3[1, 0, :] = -1
    idx3[1, 0, :len(kept)] = kept
    cnt3[1, 0] = len(kept)
    keys3, group3 = gu.block_keys(idx3, cnt3, N)
    r0 = np.arange(128)
    Os3, Ls3 = gu.oracle_rows(q, k, v, d ** -0.5, r0, [1], keys3, group3)
    gu.compare_rows(o2, lse2, Os3, Ls3, r0, "skipped entry")


def test_720p_losa_selection(bsa):
    """LoSA selection on the 720p workload's inputs (full size): dense step, mass, select."""
    wl = WORKLOADS["720p_14b"]
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    o, lse, mass = bsa.attn_dense_blockmass(q, k, v, 128, wl.scale)
    idx, cnt = bsa.losa_select(mass, wl.tau)
    assert bsa.get_device_status() == bsa.BSA_OK
    nB = mass.shape[1]
    sums = mass.double().sum(dim=2).cpu().numpy()
    assert np.abs(sums / rows_in_block(wl.N, nB)[None, :] - 1.0).max() < 1e-4
    rng = np.random.default_rng(12)
    mh = mass.cpu().numpy()
    ih, ch = idx.cpu().numpy(), cnt.cpu().numpy()
    for _ in range(400):
        h, qb = int(rng.integers(0, wl.H)), int(rng.integers(0, nB))
        ref = olosa.select_row_fast(mh[h, qb], wl.tau)
        assert ch[h, qb] == len(ref) and np.array_equal(ih[h, qb, :len(ref)], ref)
        assert np.all(ih[h, qb, len(ref):] == -1)
