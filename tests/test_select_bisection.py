"""The search the LoSA selection kernel runs for rows of up to 2048 blocks,
replayed in numpy on the CPU and checked against the oracle's selection.

The kernel does not sort.  It bisects over the 31 bits of the float mass
for the largest u with S(u) = sum of Q over blocks whose mass bits are >= u
still reaching the threshold, takes Qp = Q of the block(s) with mass bits u,
keeps every block with Q > Qp and the first ceil((threshold - A) / Qp)
blocks with Q == Qp in ascending kb (A = sum of Q over Q > Qp).  The replay
also asserts the two facts the kernel relies on without checking:
threshold > A (at least one tied block is needed) and that many tied blocks
exist.  Rows are built so that many distinct masses share one Q value
(masses below 2^-9), which is where ordering by mass and ordering by Q
differ."""
import numpy as np
import pytest

from oracle import losa as olosa


def kernel_search(m, tau):
    m = np.asarray(m, dtype=np.float32)
    q = np.floor(m.astype(np.float64) * 2.0 ** 33).astype(np.uint64)
    bits = m.view(np.uint32) & np.uint32(0x7FFFFFFF)
    total = int(q.sum())
    thr = int(np.ceil(np.float64(tau) * np.float64(total)))
    if thr == 0:
        qp, take = int(q.max()), 1
    else:
        u = 0
        for b in range(30, -1, -1):
            c = u | (1 << b)
            if int(q[bits >= c].sum()) >= thr:
                u = c
        qp = int(q[bits == u].max())
        above = int(q[q > qp].sum())
        assert thr > above                      # at least one block with Q == qp is needed
        take = (thr - above + qp - 1) // qp
    keep = q > qp
    ties = np.nonzero(q == qp)[0]               # ascending kb
    assert take <= len(ties)
    keep[ties[:take]] = True
    return np.nonzero(keep)[0]


def rows(rng, nKB):
    yield (rng.random(nKB) * 128).astype(np.float32)
    yield (rng.integers(0, 4, nKB) * 0.25).astype(np.float32)                          # exact ties
    yield ((rng.integers(0, 4, nKB) + rng.random(nKB)) * 2.0 ** -33).astype(np.float32)  # Q collisions
    yield (np.exp(rng.normal(0, 6, nKB)) % 100).astype(np.float32)                    # wide range
    z = np.zeros(nKB, np.float32)
    yield z                                                                           # all zero
    z = z.copy()
    z[rng.integers(0, nKB)] = 0.5
    yield z                                                                           # one block
    w = ((rng.integers(0, 3, nKB) + rng.random(nKB)) * 2.0 ** -33).astype(np.float32)
    w[:: 5] = 2.0 ** -20
    w[1:: 7] = -0.0
    yield w                                                                           # mixed, -0.0


@pytest.mark.parametrize("nKB", [1, 2, 3, 7, 32, 100, 256])
def test_search_matches_oracle(nKB):
    rng = np.random.default_rng(7 + nKB)
    for rep in range(12):
        for m in rows(rng, nKB):
            for tau in (0.99, 0.5, 1.0, 0.999999, 1e-9):
                got = kernel_search(m, tau)
                ref_idx, ref_cnt = olosa.select(m[None, None, :], tau)
                assert np.array_equal(got, ref_idx[0, 0, :ref_cnt[0, 0]]), (nKB, rep, tau)


def test_collision_rows_really_collide():
    """The collision rows hold many distinct masses but few distinct Q values."""
    rng = np.random.default_rng(3)
    m = list(rows(rng, 256))[2]
    q = np.floor(m.astype(np.float64) * 2.0 ** 33)
    assert len(np.unique(m)) > 200 and len(np.unique(q)) <= 4
