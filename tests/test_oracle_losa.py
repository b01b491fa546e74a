"""Oracle pins: LoSA minimal-mass selection (CPU only)."""
import numpy as np
import pytest

from oracle import losa
from tests import pins


def test_golden_hand_derived():
    pins.check_losa_golden(losa)


def test_bruteforce_subsets():
    pins.check_losa_bruteforce(losa)


def test_properties():
    pins.check_losa_properties(losa)


def test_tau_one_keeps_nonzero():
    rng = np.random.default_rng(1)
    m = (rng.random(50) * (rng.random(50) > 0.5)).astype(np.float32)
    kept = list(losa.select_row_fast(m, 1.0))
    assert kept == [i for i in range(50) if m[i] > 0]


def test_whole_tensor_layout():
    rng = np.random.default_rng(2)
    mass = rng.random((2, 3, 5)).astype(np.float32)
    idx, cnt = losa.select(mass, 0.9)
    for h in range(2):
        for qb in range(3):
            kept = losa.select_row(mass[h, qb], 0.9)
            assert cnt[h, qb] == len(kept)
            assert list(idx[h, qb, :len(kept)]) == kept
            assert np.all(idx[h, qb, len(kept):] == -1)


@pytest.mark.parametrize("bad", [-1.0, float("nan"), float("inf"), 2.0 ** 14])
def test_rejects_bad_mass(bad):
    with pytest.raises(ValueError):
        losa.select_row(np.array([0.5, bad], dtype=np.float32), 0.99)
    with pytest.raises(ValueError):
        losa.select_row_fast(np.array([0.5, bad], dtype=np.float32), 0.99)
