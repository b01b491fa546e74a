"""Oracle pins: LVSA anchors, attended-frame sets and tile lists (CPU only)."""
import pytest

import oracle
from oracle import lvsa, tiles
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS
from tests import pins


def test_golden_hand_derived_T8():
    pins.check_lvsa_golden(lvsa)


@pytest.mark.parametrize("T,T_per", [(8, 4), (21, 5), (126, 6), (126, 21), (63, 6), (7, 10), (5, 1)])
def test_anchor_coverage(T, T_per):
    pins.check_anchor_coverage(lvsa, T, T_per)


def test_bruteforce_T8():
    pins.check_lvsa_bruteforce(lvsa)


@pytest.mark.parametrize("name", ["tiny", "wan1.3b_1x_dense", "wan1.3b_1x_c11", "wan1.3b_6x",
                                  "wan1.3b_6x_tper21", "720p_14b"])
def test_invariants(name):
    wl = WORKLOADS[name]
    pins.check_lvsa_invariants(lvsa, wl.T, wl.T_per, wl.W, wl.C, range(wl.steps))


def test_budget_table():
    # |G_s| per step and the budget outcome for the workloads
    assert [len(lvsa.anchor_frames(21, 5, s)) for s in range(5)] == [5, 4, 4, 4, 4]
    assert all(len(lvsa.anchor_frames(126, 6, s)) == 21 for s in range(6))
    # 6x workload: 21 anchors already fill the budget, so non-anchor frames are over it
    A, over = lvsa.attended_frames(126, 6, 15, 21, 0)
    assert over and sorted({len(a) for a in A}) == [21, 22]
    # balanced variant: 6 anchors + 15 window frames = 21 for every t and s
    for s in range(21):
        A, over = lvsa.attended_frames(126, 21, 15, 21, s)
        assert not over and all(len(a) == 21 for a in A)
    # C >= T gives every frame (dense)
    A, over = lvsa.attended_frames(21, 5, 7, 21, 3)
    assert not over and all(a == list(range(21)) for a in A)


def test_tiles_bruteforce():
    pins.check_tiles_vs_bruteforce(tiles, lvsa)


def test_tiles_dense_full():
    # every tile kept; only tiles reaching past N are partial
    A, _ = lvsa.attended_frames(21, 5, 7, 21, 0)
    N = 21 * 1560
    idx, flg = tiles.kept_tiles(A, 21, N)
    nB = -(-N // 128)
    assert all(r == list(range(nB)) for r in idx)
    assert all(f == [0] * (nB - 1) + [1] for f in flg)


def test_pair_count_closed_form():
    # sum over query frames of |A(t)| * P^2 equals the count from the explicit mask
    for s in range(4):
        A, _ = lvsa.attended_frames(8, 4, 3, 4, s)
        m = lvsa.dense_token_mask(A, 64, 512)
        assert tiles.exact_pair_count(A, 8, 512) == int(m.sum())


def test_window_golden_hand_derived_T8():
    pins.check_lvsa_window_golden(lvsa)


def test_window_bruteforce_T8():
    pins.check_lvsa_window_bruteforce(lvsa)


@pytest.mark.parametrize("T,T_per,W", [(8, 4, 3), (21, 5, 7), (126, 6, 15), (126, 21, 15), (63, 6, 15), (5, 9, 7)])
def test_window_invariants(T, T_per, W):
    pins.check_lvsa_window_invariants(lvsa, T, T_per, W, range(min(T_per, 8) + 1))
