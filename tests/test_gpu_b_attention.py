"""GPU parity: block-sparse attention forward vs the fp64 oracle (C ABI path)."""
import math

import numpy as np
import pytest
import torch

from oracle import attention as oatt
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


def frames_tensors(A, T):
    frames = torch.full((T, T), -1, dtype=torch.int32)
    counts = torch.zeros(T, dtype=torch.int32)
    for t, a in enumerate(A):
        frames[t, :len(a)] = torch.tensor(a, dtype=torch.int32)
        counts[t] = len(a)
    return frames.cuda(), counts.cuda()


def run_lvsa(bsa, q, k, v, T, A, scale):
    frames, counts = frames_tensors(A, T)
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(T, frames, counts), scale=scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    return o, lse


def full_compare(o, lse, q, k, v, mask, scale, what, stress=False):
    """Compare every output.  Workload scale: max/mean-abs tolerance.  stress=True
    (softmax scale other than d^-1/2, very peaked rows): elementwise bound from
    bf16 rounding, |err| <= 2^-8 (|O| + sum_k p_k |v_k|) + 1e-3, i.e. twice the
    half-ulp of the bf16 output plus twice the half-ulp of the bf16 probabilities."""
    qn, kn, vn = (x.cpu().to(torch.float64).numpy() for x in (q, k, v))
    O, L = oatt.attention_dense_masked(qn, kn, vn, scale, mask)
    og = o.cpu().to(torch.float64).numpy()
    lg = lse.cpu().to(torch.float64).numpy()
    err = np.abs(og - O)
    if stress:
        Oabs, _ = oatt.attention_dense_masked(qn, kn, np.abs(vn), scale, mask)
        bound = 2.0 ** -8 * (np.abs(O) + Oabs) + 1e-3
        assert np.all(err <= bound), f"{what}: worst err/bound {(err / bound).max()}"
    else:
        assert err.max() <= gu.O_MAX, f"{what}: O max {err.max()}"
        assert err.mean() <= gu.O_MEAN, f"{what}: O mean {err.mean()}"
    fin = np.isfinite(L)
    assert np.array_equal(fin, np.isfinite(lg)), what
    if fin.any():
        assert np.abs(lg[fin] - L[fin]).max() <= gu.LSE_MAX, what


def test_tiny_all_steps(bsa):
    wl = WORKLOADS["tiny"]
    for s in range(wl.steps):
        q, k, v = inputs.workload_qkv(wl, s, device="cuda")
        frames, counts, over = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, device="cuda")
        o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(wl.T, frames, counts), scale=wl.scale)
        assert bsa.get_device_status() == bsa.BSA_OK
        A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, s)
        full_compare(o, lse, q, k, v, olvsa.dense_token_mask(A, wl.P, wl.N), wl.scale, f"tiny s={s}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("T,P", [(5, 100), (7, 37), (3, 200), (2, 300), (9, 29), (4, 128), (1, 77), (6, 129)])
def test_ragged_lvsa(bsa, d, T, P):
    N, H = T * P, 3
    rng = np.random.default_rng(T * 1000 + P)
    q, k, v = inputs.make_qkv(N, H, d, seed=T * 7 + P, device="cuda")
    C = int(rng.integers(1, T + 1))
    s = int(rng.integers(0, 10))
    A, _ = olvsa.attended_frames(T, max(1, T // 2), 1, C, s)
    o, lse = run_lvsa(bsa, q, k, v, T, A, d ** -0.5)
    full_compare(o, lse, q, k, v, olvsa.dense_token_mask(A, P, N), d ** -0.5, f"ragged T={T} P={P} d={d}")


def test_arbitrary_frame_sets(bsa):
    rng = np.random.default_rng(5)
    T, P, d, H = 6, 90, 128, 2
    N = T * P
    q, k, v = inputs.make_qkv(N, H, d, seed=77, device="cuda")
    for trial in range(4):
        A = [sorted({t} | {f for f in range(T) if rng.random() < 0.3}) for t in range(T)]
        o, lse = run_lvsa(bsa, q, k, v, T, A, d ** -0.5)
        full_compare(o, lse, q, k, v, olvsa.dense_token_mask(A, P, N), d ** -0.5, f"arbitrary {trial}")
        o, lse = run_lvsa(bsa, q, k, v, T, A, 0.2)
        full_compare(o, lse, q, k, v, olvsa.dense_token_mask(A, P, N), 0.2, f"arbitrary {trial} s=0.2",
                     stress=True)


def test_large_logits_rescale(bsa):
    # scores spread over many units: exercises the running-max rescale of O
    T, P, d, H = 4, 256, 64, 2
    N = T * P
    q, k, v = inputs.make_qkv(N, H, d, seed=3, device="cuda")
    A = [list(range(T)) for _ in range(T)]
    for scale in (1.0, 0.5, 0.0):
        o, lse = run_lvsa(bsa, q, k, v, T, A, scale)
        full_compare(o, lse, q, k, v, olvsa.dense_token_mask(A, P, N), scale, f"scale={scale}", stress=True)


def test_closed_forms(bsa):
    T, P, d, H = 8, 64, 64, 2
    N = T * P
    A, _ = olvsa.attended_frames(T, 4, 3, 4, 1)
    mask = olvsa.dense_token_mask(A, P, N)
    q, k, v = inputs.make_qkv(N, H, d, seed=9, device="cuda")
    # v == c  =>  O == c (0.375 is exact in bf16)
    vc = torch.full_like(v, 0.375)
    o, _ = run_lvsa(bsa, q, k, vc, T, A, 0.125)
    assert torch.all(o.float() == 0.375)
    # q == 0  =>  O = mean of the allowed v rows, LSE = log(#allowed)
    o, lse = run_lvsa(bsa, torch.zeros_like(q), k, v, T, A, 0.125)
    vn = v.cpu().double().numpy()
    for r in (0, 63, 64, 300, 511):
        keys = np.nonzero(mask[r])[0]
        ref = vn[keys].mean(axis=0)
        assert np.abs(o[r].cpu().double().numpy() - ref).max() < 5e-3
        assert abs(lse[0, r].item() - math.log(len(keys))) < 1e-4


def sampled_lvsa(bsa, wl, s, rows_n, heads, seed):
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    frames, counts, _ = bsa.lvsa_build_index(wl.T, wl.T_per, wl.W, wl.C, s, device="cuda")
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(wl.T, frames, counts), scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, s)
    rows = inputs.sample_rows(wl.N, wl.P, rows_n, seed).numpy()
    keys, group = gu.lvsa_keys(A, wl.P, wl.N)
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, heads, keys, group)
    return gu.compare_rows(o, lse, Os, Ls, rows, f"{wl.name} s={s}")


def test_wan_1x_dense_budget(bsa):
    sampled_lvsa(bsa, WORKLOADS["wan1.3b_1x_dense"], 0, 160, [0, 11], 21)


def test_wan_1x_c11(bsa):
    for s in (0, 1):
        sampled_lvsa(bsa, WORKLOADS["wan1.3b_1x_c11"], s, 160, [0, 5], 22 + s)


@pytest.mark.parametrize("s", [0, 1, 39])
def test_wan_6x_full_size(bsa, s):
    sampled_lvsa(bsa, WORKLOADS["wan1.3b_6x"], s, 192, [0, 7, 11], 30 + s)


def test_wan_6x_balanced(bsa):
    sampled_lvsa(bsa, WORKLOADS["wan1.3b_6x_tper21"], 2, 128, [3], 40)


@pytest.mark.parametrize("name,s", [("wan1.3b_1x_c11", 0), ("wan1.3b_1x_c11", 3), ("wan1.3b_6x", 1)])
def test_window_reading(bsa, name, s):
    """Attention on the fixed-window frame sets (|A(t)| = |G_s| + W)."""
    wl = WORKLOADS[name]
    q, k, v = inputs.workload_qkv(wl, s, device="cuda")
    frames, counts = bsa.lvsa_build_index_window(wl.T, wl.T_per, wl.W, s, device="cuda")
    o, lse = bsa.blocksparse_attn_fwd(q, k, v, bsa.lvsa_index(wl.T, frames, counts), scale=wl.scale)
    assert bsa.get_device_status() == bsa.BSA_OK
    A = olvsa.attended_frames_window(wl.T, wl.T_per, wl.W, s)
    rows = inputs.sample_rows(wl.N, wl.P, 128, 60 + s).numpy()
    keys, group = gu.lvsa_keys(A, wl.P, wl.N)
    Os, Ls = gu.oracle_rows(q, k, v, wl.scale, rows, [0, 5], keys, group)
    gu.compare_rows(o, lse, Os, Ls, rows, f"{name} window s={s}")


def test_720p_lvsa_full_size(bsa):
    sampled_lvsa(bsa, WORKLOADS["720p_14b"], 0, 128, [0, 39], 50)


@pytest.mark.parametrize("name,s", [("hunyuan1.5_1.5x", 0), ("hunyuan1.5_2x", 0), ("hunyuan1.5_2x", 5)])
def test_hunyuan_horizons_full_size(bsa, name, s):
    """HunyuanVideo-1.5-shaped long video at 1.5x and 2x its training horizon."""
    sampled_lvsa(bsa, WORKLOADS[name], s, 128, [0, 15], 55 + s)
