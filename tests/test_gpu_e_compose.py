"""GPU parity: LoSA's block selection inside LVSA's frame sets - the block
mass of LVSA-restricted attention, the selection made from it, and the
intersection index (LVSA element rule within the selected key blocks)."""
import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import losa as olosa
from oracle import lvsa as olvsa
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
from block_sparse_attention_lvsa_b200 import inputs
from tests import gpu_util as gu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


@pytest.fixture(scope="module")
def case(bsa):
    """LVSA step 1 of the Wan-1.3B shape at C = 11, its restricted mass and selection."""
    wl = WORKLOADS["wan1.3b_1x_c11"]
    s = 1
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, device="cuda")
    ix = bsa.lvsa_index(wl.T, frames, counts)
    o, lse, mass = bsa.attn_blockmass(q, k, v, ix, wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    idx, cnt = bsa.losa_select(mass, 0.99)
    assert bsa.get_device_status() == bsa.BSA_OK
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, s)
    return dict(wl=wl, qkv=(q, k, v), frames=frames, counts=counts, ix=ix, o=o, lse=lse, mass=mass,
                idx=idx, cnt=cnt, A=A)


def test_restricted_outputs_equal_forward(bsa, case):
    """Mass mode adds stores only: O and LSE equal the plain forward bit for bit."""
    q, k, v = case["qkv"]
    o2, lse2 = bsa.blocksparse_attn_fwd(q, k, v, case["ix"], scale=case["wl"].scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(case["o"], o2) and torch.equal(case["lse"], lse2)


def test_restricted_mass_vs_oracle(bsa, case):
    wl, A = case["wl"], case["A"]
    q, k, _ = case["qkv"]
    mg = case["mass"].cpu().double().numpy()
    nB = mg.shape[1]
    # rows of every block sum to the block's row count; blocks LVSA never reaches hold 0
    rows = np.array([min((b + 1) * 128, wl.N) - b * 128 for b in range(nB)], dtype=np.float64)
    assert np.abs(mg.sum(axis=2) / rows[None, :] - 1.0).max() <= 1e-5
    heads, qblocks = [0, 7], [0, 17, 128, nB - 1]
    for h in heads:
        qh, kh = gu.head_f64(q, h), gu.head_f64(k, h)
        ref = oatt.block_mass_restricted(qh, kh, wl.scale, 128, [0], qblocks,
                                         lambda _h, r: olvsa.allowed_keys_for_row(r, A, wl.P, wl.N))
        for qb in qblocks:
            e = np.abs(mg[h, qb] - ref[(0, qb)]).max() / rows[qb]
            assert e <= gu.MASS_MAX, (h, qb, e)
            assert np.all(mg[h, qb][ref[(0, qb)] == 0.0] == 0.0)


def test_dense_index_mass_equals_dense_blockmass(bsa):
    """With every frame allowed the restricted mass is the dense measuring step, bit for bit."""
    wl = WORKLOADS["wan1.3b_1x_dense"]
    q, k, v = inputs.workload_qkv(wl, 0, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.T, 0, device="cuda")
    o1, l1, m1 = bsa.attn_blockmass(q, k, v, bsa.lvsa_index(wl.T, frames, counts), wl.scale)
    o2, l2, m2 = bsa.attn_dense_blockmass(q, k, v, 128, wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o1, o2) and torch.equal(l1, l2) and torch.equal(m1, m2)


def test_selection_inside_lvsa(bsa, case):
    """Bit-exact against the oracle on the GPU mass; every kept block is one LVSA keeps."""
    idx, cnt = case["idx"].cpu().numpy(), case["cnt"].cpu().numpy()
    ref_idx, ref_cnt = olosa.select(case["mass"].cpu().numpy(), 0.99)
    assert np.array_equal(cnt, ref_cnt) and np.array_equal(idx, ref_idx)
    wl, A = case["wl"], case["A"]
    from oracle import tiles as otiles
    lv, _ = otiles.kept_tiles(A, wl.T, wl.N)
    for qb in range(cnt.shape[1]):
        allowed = set(lv[qb])
        for h in range(cnt.shape[0]):
            assert set(idx[h, qb, :cnt[h, qb]].tolist()) <= allowed, (h, qb)
    # the selection is sparser than LVSA alone
    assert cnt.sum() < cnt.shape[0] * sum(len(x) for x in lv)


def test_intersection_with_all_blocks_is_lvsa(bsa, case):
    """Every block listed: the intersection is LVSA alone, bit for bit (tiles LVSA
    does not keep are fully masked and add exact zeros)."""
    wl = case["wl"]
    q, k, v = case["qkv"]
    H, nB = case["mass"].shape[0], case["mass"].shape[1]
    idx = torch.arange(nB, dtype=torch.int32, device="cuda").repeat(H, nB, 1).contiguous()
    cnt = torch.full((H, nB), nB, dtype=torch.int32, device="cuda")
    ix3 = bsa.lvsa_block_index(wl.T, case["frames"], case["counts"], idx, cnt)
    o3, l3 = bsa.blocksparse_attn_fwd(q, k, v, ix3, scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    assert torch.equal(o3, case["o"]) and torch.equal(l3, case["lse"])


def test_intersection_vs_oracle(bsa, case):
    wl, A = case["wl"], case["A"]
    q, k, v = case["qkv"]
    ix3 = bsa.lvsa_block_index(wl.T, case["frames"], case["counts"], case["idx"], case["cnt"])
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, ix3, scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    idx, cnt = case["idx"].cpu().numpy(), case["cnt"].cpu().numpy()
    block_keys, _ = gu.block_keys(idx, cnt, wl.N)

    def keys(h, r):
        return np.intersect1d(olvsa.allowed_keys_for_row(r, A, wl.P, wl.N), block_keys(h, r))

    rows = inputs.sample_rows(wl.N, wl.P, 128, 77).numpy()
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, [0, 9], keys, None)
    gu.compare_rows(o, lse, Os, Ls, rows, "LVSA within LoSA blocks")
