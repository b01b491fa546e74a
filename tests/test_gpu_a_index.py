"""GPU parity: LVSA index build and the tile-list expansion, bit-exact vs the oracle."""
import numpy as np
import pytest
import torch

from oracle import lvsa as olvsa
from oracle import tiles as otiles
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS

pytestmark = pytest.mark.gpu

LVSA_WL = ["tiny", "wan1.3b_1x_dense", "wan1.3b_1x_c11", "wan1.3b_6x", "wan1.3b_6x_tper21", "720p_14b",
           "hunyuan1.5_1.5x", "hunyuan1.5_2x"]


@pytest.fixture(scope="module")
def bsa():
    from block_sparse_attention_lvsa_b200 import binding
    assert torch.cuda.is_available()
    return binding


def check_index(bsa, T, T_per, W, C, s):
    frames, counts, over = bsa.lvsa_build_index(T, T_per, W, C, s, device="cuda")
    A, over_ref = olvsa.attended_frames(T, T_per, W, C, s)
    fr = frames.cpu().numpy()
    ct = counts.cpu().numpy()
    assert over == over_ref, (T, T_per, C, s)
    for t in range(T):
        assert ct[t] == len(A[t]), (T, T_per, C, s, t)
        assert list(fr[t, :ct[t]]) == A[t], (T, T_per, C, s, t)
        assert np.all(fr[t, ct[t]:] == -1)


@pytest.mark.parametrize("name", LVSA_WL)
def test_build_index_workloads(bsa, name):
    wl = WORKLOADS[name]
    for s in sorted(set(list(range(wl.T_per + 1)) + [wl.steps - 1])):
        check_index(bsa, wl.T, wl.T_per, wl.W, wl.C, s)


def test_build_index_random(bsa):
    rng = np.random.default_rng(0)
    for _ in range(60):
        T = int(rng.integers(1, 300))
        T_per = int(rng.integers(1, 40))
        C = int(rng.integers(1, T + 3))
        s = int(rng.integers(0, 100))
        check_index(bsa, T, T_per, 1, C, s)
    check_index(bsa, 1024, 7, 3, 50, 5)     # largest supported T
    check_index(bsa, 1, 1, 1, 1, 0)         # degenerate single frame


def check_window_index(bsa, T, T_per, W, s):
    frames, counts = bsa.lvsa_build_index_window(T, T_per, W, s, device="cuda")
    A = olvsa.attended_frames_window(T, T_per, W, s)
    fr = frames.cpu().numpy()
    ct = counts.cpu().numpy()
    for t in range(T):
        assert ct[t] == len(A[t]), (T, T_per, W, s, t)
        assert list(fr[t, :ct[t]]) == A[t], (T, T_per, W, s, t)
        assert np.all(fr[t, ct[t]:] == -1)


@pytest.mark.parametrize("name", LVSA_WL)
def test_window_index_workloads(bsa, name):
    """Fixed-window reading, bit-exact vs the oracle, every anchor phase."""
    wl = WORKLOADS[name]
    for s in sorted(set(list(range(wl.T_per + 1)) + [wl.steps - 1])):
        check_window_index(bsa, wl.T, wl.T_per, wl.W, s)


def test_window_index_random(bsa):
    rng = np.random.default_rng(1)
    for _ in range(60):
        T = int(rng.integers(1, 300))
        check_window_index(bsa, T, int(rng.integers(1, 40)), int(rng.integers(1, T + 3)), int(rng.integers(0, 100)))
    check_window_index(bsa, 1024, 7, 30, 5)
    check_window_index(bsa, 1, 1, 1, 0)


def tile_lists(bsa, T, P, A, d=64):
    """Run the forward once (H=1) and decode the tile lists from the workspace."""
    N = T * P
    frames = torch.full((T, T), -1, dtype=torch.int32)
    counts = torch.zeros(T, dtype=torch.int32)
    for t, a in enumerate(A):
        frames[t, :len(a)] = torch.tensor(a, dtype=torch.int32)
        counts[t] = len(a)
    frames, counts = frames.cuda(), counts.cuda()
    q = torch.zeros((N, 1, d), dtype=torch.bfloat16, device="cuda")
    ix = bsa.lvsa_index(T, frames, counts)
    ws = torch.empty(bsa.workspace_bytes(bsa.BSA_OP_BLOCKSPARSE_FWD, N, 1, d, ix), dtype=torch.uint8, device="cuda")
    bsa.blocksparse_attn_fwd(q, q, q, ix, workspace=ws)
    assert bsa.get_device_status() == bsa.BSA_OK
    _, cnt, idx, flag = bsa.lvsa_workspace_views(ws, N, T)
    return cnt.cpu().numpy(), idx.cpu().numpy(), flag.cpu().numpy()


def compare_tiles(cnt, idx, flag, ref_idx, ref_flg, qtiles):
    for i, qt in enumerate(qtiles):
        n = cnt[qt]
        assert n == len(ref_idx[i]), qt
        assert list(idx[qt, :n]) == ref_idx[i], qt
        assert list(flag[qt, :n]) == ref_flg[i], qt


def test_tiles_small_random(bsa):
    rng = np.random.default_rng(1)
    for T, P in [(8, 64), (5, 100), (7, 37), (3, 200), (2, 300), (9, 29), (4, 128), (1, 77)]:
        for trial in range(3):
            A = [sorted({t} | {f for f in range(T) if rng.random() < 0.4}) for t in range(T)]
            cnt, idx, flag = tile_lists(bsa, T, P, A)
            ri, rf = otiles.kept_tiles(A, T, T * P)
            compare_tiles(cnt, idx, flag, ri, rf, range(len(ri)))


@pytest.mark.parametrize("name,steps", [("tiny", [0, 1, 2, 3]), ("wan1.3b_1x_c11", [0, 3]),
                                        ("wan1.3b_6x", [0, 5]), ("720p_14b", [0]),
                                        ("hunyuan1.5_1.5x", [0, 1]), ("hunyuan1.5_2x", [0, 5])])
def test_tiles_workloads(bsa, name, steps):
    wl = WORKLOADS[name]
    nB = -(-wl.N // 128)
    rng = np.random.default_rng(2)
    qtiles = sorted(set([0, nB - 1] + rng.integers(0, nB, 48).tolist())) if nB > 64 else list(range(nB))
    for s in steps:
        A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, s)
        cnt, idx, flag = tile_lists(bsa, wl.T, wl.P, A)
        ri, rf = otiles.kept_tiles(A, wl.T, wl.N, qtiles=qtiles)
        compare_tiles(cnt, idx, flag, ri, rf, qtiles)
