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


def large_total_row(n_zero: int) -> np.ndarray:
    """256 blocks of mass 2^13 (Q = 2^46 each, sum 2^54), one block of mass
    3 * 2^-33 (Q = 3) and `n_zero` empty blocks: the row total 2^54 + 3 is
    not a float64 and rounds up to 2^54 + 4 when converted."""
    m = np.zeros(257 + n_zero, dtype=np.float32)
    m[:256] = 2.0 ** 13
    m[256] = 3 * 2.0 ** -33
    perm = np.random.default_rng(3).permutation(m.size)
    return m[perm]


@pytest.mark.parametrize("n_zero", [0, 43, 2000])
def test_tau_one_large_total(n_zero):
    # At tau = 1 the minimal set holding the whole mass is exactly the set of
    # blocks with positive mass, whatever the float64 rounding of the total.
    m = large_total_row(n_zero)
    total = 256 * 2 ** 46 + 3
    assert float(total) > total                      # the case the clamp is for
    want = [i for i in range(m.size) if m[i] > 0]
    assert losa.select_row(m, 1.0) == want
    assert list(losa.select_row_fast(m, 1.0)) == want
