"""The search the LoSA selection kernel runs for rows of up to 512 blocks,
replayed in plain Python integers on the CPU and checked against the
oracle's selection.

The kernel does not sort.  It bisects over the 31 bits of the float mass
for the largest u with S(u) = sum of Q over blocks whose mass bits are >= u
still reaching the threshold, stopping early once the remaining interval
[u, u + 2^b) holds blocks of a single mass value (that value is then u; the
check runs after the rounds of bits 24, 21, ..., 3).  It takes Qp = Q of the
block(s) with mass bits u, keeps every block with Q > Qp and the first
ceil((threshold - A) / Qp) blocks with Q == Qp in ascending kb (A = sum of Q
over Q > Qp).  The replay asserts the facts the kernel relies on without
checking: threshold > A (at least one tied block is needed), that many tied
blocks exist, and the interval invariant S(u) >= threshold > S(u + 2^b) at
every early-exit check (some block lies in the interval).  Rows are built so
that many distinct masses share one Q value (masses below 2^-9), which is
where ordering by mass and ordering by Q differ."""
import math

import numpy as np
import pytest

from oracle import losa as olosa

EXIT_CHECKS = (24, 21, 18, 15, 12, 9, 6, 3)     # bits after whose round the kernel tries the early exit


def kernel_search(m, tau, stats=None):
    m = np.asarray(m, dtype=np.float32)
    bits = [int(b) & 0x7FFFFFFF for b in m.view(np.uint32)]
    q = [math.floor(math.ldexp(float(x), 33)) for x in m.tolist()]
    total = sum(q)

    def row_sum(sel):
        return sum(q[i] for i in sel)

    n = len(m)
    thr = min(math.ceil(float(tau) * float(total)), total)
    rounds = 0
    if thr == 0:
        qp, take = max(q), 1
    else:
        u = 0
        for b in range(30, -1, -1):
            c = u | (1 << b)
            rounds += 1
            if row_sum([i for i in range(n) if bits[i] >= c]) >= thr:
                u = c
            if b in EXIT_CHECKS:
                inside = [bits[i] for i in range(n) if u <= bits[i] < u + (1 << b)]
                assert inside                          # S(u) >= thr > S(u + 2^b)
                if min(inside) == max(inside):
                    u = inside[0]
                    break
        qp = max(q[i] for i in range(n) if bits[i] == u)
        above = row_sum([i for i in range(n) if q[i] > qp])
        assert thr > above                          # at least one block with Q == qp is needed
        take = (thr - above + qp - 1) // qp
    ties = [i for i in range(n) if q[i] == qp]      # ascending kb
    assert take <= len(ties)
    keep = sorted([i for i in range(n) if q[i] > qp] + ties[:take])
    if stats is not None:
        stats.append(rounds)
    return np.asarray(keep, dtype=np.int64)


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
    big = (rng.random(nKB) * 16383).astype(np.float32)                                # totals above 2^48
    yield big


def softmax_like(rng, nKB):
    """Block masses shaped like a measuring step's: lognormal weights normalised to 128 rows."""
    w = np.exp(rng.normal(0, 2.5, nKB))
    return (w / w.sum() * 128).astype(np.float32)


@pytest.mark.parametrize("nKB", [1, 2, 3, 7, 32, 100, 256, 600])
def test_search_matches_oracle(nKB):
    rng = np.random.default_rng(7 + nKB)
    reps = 12 if nKB <= 256 else 3
    for rep in range(reps):
        for m in list(rows(rng, nKB)) + [softmax_like(rng, nKB)]:
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


def test_early_exit_shortens_typical_rows():
    """On measuring-step-shaped rows the search ends well before 31 rounds."""
    rng = np.random.default_rng(11)
    stats = []
    for _ in range(40):
        kernel_search(softmax_like(rng, 256), 0.99, stats)
    assert np.mean(stats) <= 20, np.mean(stats)
