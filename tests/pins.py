"""Checks that pin the oracle to facts fixed outside it.

Each check takes the oracle module(s) as an argument so the same check can
be run against the real oracle (must pass) and against an oracle with a
planted mistake (must fail).  None of them re-types an oracle formula: they
compare with hand-derived fixtures, closed forms, invariants, library
routines on special cases, or brute-force enumeration.
"""
from __future__ import annotations

import itertools
import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------- LVSA ----
def read_lvsa_golden():
    table = {}
    with open(os.path.join(GOLDEN, "lvsa_T8_Tper4_C4.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, frames = line.split(":")
            s, t = map(int, head.split())
            table[(s, t)] = [int(x) for x in frames.split()]
    return table


def check_lvsa_golden(lvsa):
    table = read_lvsa_golden()
    for s in range(4):
        A, over = lvsa.attended_frames(8, 4, 3, 4, s)
        assert not over
        for t in range(8):
            assert A[t] == table[(s, t)], (s, t, A[t], table[(s, t)])


def check_anchor_coverage(lvsa, T, T_per, start_steps=(0, 1, 7, 40)):
    """Every frame is an anchor exactly once over any T_per consecutive steps."""
    for s0 in start_steps:
        seen = [0] * T
        for s in range(s0, s0 + T_per):
            for f in lvsa.anchor_frames(T, T_per, s):
                seen[f] += 1
        assert all(c == 1 for c in seen), (T, T_per, s0, seen)


def brute_force_A(T, T_per, C, s, anchors_fn):
    """Lexicographically smallest size-C superset of G_s u {t} under (distance, frame) order.

    Enumerates every subset of the non-base frames of the required size and
    keeps the one whose sorted (|f - t|, f) key tuple is smallest.
    """
    G = set(anchors_fn(T, T_per, s))
    out = []
    for t in range(T):
        base = G | {t}
        if len(base) >= C:
            out.append(sorted(base))
            continue
        rest = [f for f in range(T) if f not in base]
        need = min(C - len(base), len(rest))
        best = None
        for X in itertools.combinations(rest, need):
            key = sorted((abs(f - t), f) for f in X)
            if best is None or key < best[0]:
                best = (key, X)
        out.append(sorted(base | set(best[1])))
    return out


def check_lvsa_bruteforce(lvsa, T=8):
    for T_per in (1, 2, 3, 4, 5, 9):
        for C in (1, 2, 3, 4, 5, 8, 11):
            for s in range(T_per + 1):
                A, _ = lvsa.attended_frames(T, T_per, 3, C, s)
                # anchors from the closed form, independent of the oracle
                ref = brute_force_A(T, T_per, C, s,
                                    lambda T_, p, s_: [f for f in range(T_) if (f - s_) % p == 0])
                assert A == ref, (T_per, C, s)


def check_lvsa_invariants(lvsa, T, T_per, W, C, steps):
    for s in steps:
        G = [f for f in range(T) if (f - s) % T_per == 0]
        A, over = lvsa.attended_frames(T, T_per, W, C, s)
        any_over = False
        for t in range(T):
            a = A[t]
            assert a == sorted(set(a)) and all(0 <= f < T for f in a)
            assert set(G) <= set(a) and t in a
            base = len(set(G) | {t})
            if base <= C:
                assert len(a) == min(C, T)
            else:
                any_over = True
                assert set(a) == set(G) | {t}
        assert over == any_over
        # depends on s only through s mod T_per
        assert A == lvsa.attended_frames(T, T_per, W, C, s % T_per)[0]


def read_lvsa_window_golden():
    table = {}
    with open(os.path.join(GOLDEN, "lvsa_window_T8_Tper4_W3.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            head, frames = line.split(":")
            s, t = map(int, head.split())
            table[(s, t)] = [int(x) for x in frames.split()]
    return table


def check_lvsa_window_golden(lvsa):
    table = read_lvsa_window_golden()
    assert len(table) == 32
    for s in range(4):
        A = lvsa.attended_frames_window(8, 4, 3, s)
        for t in range(8):
            assert A[t] == table[(s, t)], (s, t, A[t], table[(s, t)])


def brute_force_window(T, T_per, W, s):
    """Fixed-window reading by exhaustive search: among all sets X of
    min(W, #non-anchors) non-anchor frames that hold t when t is not an
    anchor, the one whose sorted (|f - t|, f) tuple is smallest."""
    G = {f for f in range(T) if (f - s) % T_per == 0}
    free = [f for f in range(T) if f not in G]
    n = min(W, len(free))
    out = []
    for t in range(T):
        best = None
        for X in itertools.combinations(free, n):
            if t not in G and t not in X:
                continue
            key = sorted((abs(f - t), f) for f in X)
            if best is None or key < best[0]:
                best = (key, X)
        out.append(sorted(G | {t} | set(best[1])))
    return out


def check_lvsa_window_bruteforce(lvsa, T=8):
    for T_per in (1, 2, 3, 4, 5, 9):
        for W in (1, 2, 3, 5, 8):
            for s in range(T_per + 1):
                assert lvsa.attended_frames_window(T, T_per, W, s) == brute_force_window(T, T_per, W, s), \
                    (T_per, W, s)


def check_lvsa_window_invariants(lvsa, T, T_per, W, steps):
    for s in steps:
        G = {f for f in range(T) if (f - s) % T_per == 0}
        A = lvsa.attended_frames_window(T, T_per, W, s)
        for t in range(T):
            a = A[t]
            assert a == sorted(set(a)) and all(0 <= f < T for f in a)
            assert G <= set(a) and t in a
            assert len(a) == len(G) + min(W, T - len(G))
        # the two readings agree once the budget is |G_s| + W (balanced configurations)
        assert A == lvsa.attended_frames(T, T_per, W, min(T, len(G) + W), s)[0]


# ---------------------------------------------------------------- tiles ---
def random_allowed(T, rng, density=0.4):
    A = []
    for t in range(T):
        fr = {t} | {f for f in range(T) if rng.random() < density}
        A.append(sorted(fr))
    return A


def check_tiles_vs_bruteforce(tiles, lvsa):
    rng = np.random.default_rng(7)
    cases = [(8, 64), (5, 100), (7, 37), (3, 200), (4, 128), (2, 300), (9, 29)]
    for T, P in cases:
        N = T * P
        for trial in range(3):
            A = random_allowed(T, rng)
            assert tiles.kept_tiles(A, T, N) == tiles.kept_tiles_bruteforce(A, T, N), (T, P)
    for s in range(4):
        A, _ = lvsa.attended_frames(8, 4, 3, 4, s)
        assert tiles.kept_tiles(A, 8, 512) == tiles.kept_tiles_bruteforce(A, 8, 512)


# ------------------------------------------------------------ attention ---
def sdpa_f64(q, k, v, scale, mask=None):
    """torch CPU float64 scaled_dot_product_attention, [N,H,d] layout in and out."""
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]
    K = torch.from_numpy(k).permute(1, 0, 2)[None]
    V = torch.from_numpy(v).permute(1, 0, 2)[None]
    am = None if mask is None else torch.from_numpy(mask)
    O = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=am, scale=scale)
    return O[0].permute(1, 0, 2).numpy()


def check_attention_vs_sdpa(attention, lvsa, rng_seed=3):
    rng = np.random.default_rng(rng_seed)
    # dense (budget covers every frame) and LVSA-masked, T=8 P=64 N=512
    N, H, d, T = 512, 2, 64, 8
    q, k, v = (rng.standard_normal((N, H, d)) for _ in range(3))
    scale = d ** -0.5
    Afull, _ = lvsa.attended_frames(T, 4, 3, 8, 0)
    O, _ = attention.attention_dense_masked(q, k, v, scale, lvsa.dense_token_mask(Afull, 64, N))
    assert np.allclose(O, sdpa_f64(q, k, v, scale), atol=1e-12, rtol=1e-10)
    A, _ = lvsa.attended_frames(T, 4, 3, 4, 1)
    mask = lvsa.dense_token_mask(A, 64, N)
    O, _ = attention.attention_dense_masked(q, k, v, scale, mask)
    assert np.allclose(O, sdpa_f64(q, k, v, scale, mask), atol=1e-12, rtol=1e-10)
    # row path with per-row key lists must agree with the library as well
    rows = [0, 63, 64, 200, 511]
    Os, _ = attention.attention_rows(q, k, v, scale, rows, range(H),
                                     lambda h, r: lvsa.allowed_keys_for_row(r, A, 64, N))
    ref = sdpa_f64(q, k, v, scale, mask)
    for h in range(H):
        assert np.allclose(Os[h], ref[rows, h, :], atol=1e-12, rtol=1e-10)


def check_attention_closed_forms(attention, lvsa):
    rng = np.random.default_rng(11)
    N, H, d, T, P = 512, 2, 64, 8, 64
    A, _ = lvsa.attended_frames(T, 4, 3, 4, 2)
    mask = lvsa.dense_token_mask(A, P, N)
    q, k = rng.standard_normal((N, H, d)), rng.standard_normal((N, H, d))
    # v == c  =>  O == c
    v = np.full((N, H, d), 0.37)
    O, _ = attention.attention_dense_masked(q, k, v, 0.125, mask)
    assert np.allclose(O, 0.37, atol=1e-13)
    # q == 0  =>  O = mean of allowed v rows, LSE = log(number of allowed keys)
    v = rng.standard_normal((N, H, d))
    q0 = np.zeros((N, H, d))
    O, L = attention.attention_dense_masked(q0, k, v, 0.125, mask)
    for r in (0, 100, 300, 511):
        allowed = np.nonzero(mask[r])[0]
        for h in range(H):
            assert np.allclose(O[r, h], v[allowed, h].mean(axis=0), atol=1e-12)
            assert abs(L[h, r] - math.log(len(allowed))) < 1e-12
    # empty row => O = 0, LSE = -inf
    m2 = mask.copy()
    m2[5, :] = False
    O, L = attention.attention_dense_masked(q, k, v, 0.125, m2)
    assert np.all(O[5] == 0) and np.all(np.isneginf(L[:, 5]))


def check_attention_triple_loop(attention, lvsa):
    """Pure-Python loops with math.exp on a few rows of the tiny workload."""
    rng = np.random.default_rng(5)
    N, H, d, T, P = 512, 2, 64, 8, 64
    q, k, v = (rng.standard_normal((N, H, d)) for _ in range(3))
    A, _ = lvsa.attended_frames(T, 4, 3, 4, 3)
    scale = 0.125
    rows = [1, 130, 449]
    Os, Ls = attention.attention_rows(q, k, v, scale, rows, range(H),
                                      lambda h, r: lvsa.allowed_keys_for_row(r, A, P, N))
    for h in range(H):
        for i, r in enumerate(rows):
            fr = A[r // P]
            keys = [kk for kk in range(N) if kk // P in fr]
            s = []
            for kk in keys:
                acc = 0.0
                for j in range(d):
                    acc += q[r, h, j] * k[kk, h, j]
                s.append(acc * scale)
            mx = max(s)
            e = [math.exp(x - mx) for x in s]
            tot = sum(e)
            for j in range(0, d, 9):
                o = sum(e[n] * v[keys[n], h, j] for n in range(len(keys))) / tot
                assert abs(o - Os[h][i, j]) < 1e-10
            assert abs(mx + math.log(tot) - Ls[h][i]) < 1e-10


def check_block_mass(attention):
    rng = np.random.default_rng(9)
    N, H, d, blk = 300, 2, 16, 128          # ragged last block (44 rows)
    q, k = rng.standard_normal((N, H, d)), rng.standard_normal((N, H, d))
    scale = 0.3
    nB = 3
    got = attention.block_mass(q, k, scale, blk, range(H), range(nB))
    for h in range(H):
        S = torch.from_numpy(q[:, h] @ k[:, h].T * scale)
        p = torch.softmax(S, dim=-1).numpy()             # library softmax
        ref = attention.block_mass_from_probabilities(p, blk)
        for qb in range(nB):
            assert np.allclose(got[(h, qb)], ref[qb], atol=1e-12)
            rows = min((qb + 1) * blk, N) - qb * blk
            assert abs(got[(h, qb)].sum() - rows) < 1e-9      # sum over kb = rows
    # q == 0: uniform probabilities, mass = rows(qb) * cols(kb) / N
    got = attention.block_mass(np.zeros_like(q), k, scale, blk, [0], range(nB))
    sizes = [128, 128, 44]
    for qb in range(nB):
        for kb in range(nB):
            assert abs(got[(0, qb)][kb] - sizes[qb] * sizes[kb] / N) < 1e-12


def check_block_mass_restricted(attention, lvsa):
    """Block mass of frame-restricted attention: the library softmax over the
    masked score matrix, summed over rectangles in the test; rows sum to 1
    (rows with an allowed key); nothing outside allowed blocks; dense sets
    give the dense mass; q = 0 gives the closed form."""
    rng = np.random.default_rng(11)
    T, P, H, d, blk = 6, 70, 2, 16, 128                 # N = 420: 4 blocks, ragged last (36 rows)
    N = T * P
    q, k = rng.standard_normal((N, H, d)), rng.standard_normal((N, H, d))
    scale = 0.35
    nB = -(-N // blk)
    edges = np.arange(0, N, blk)
    for dense in (False, True):
        A = [list(range(T))] * T if dense else random_allowed(T, rng, 0.3)
        mask = lvsa.dense_token_mask(A, P, N)
        allowed = lambda h, r: lvsa.allowed_keys_for_row(r, A, P, N)     # noqa: E731
        got = attention.block_mass_restricted(q, k, scale, blk, range(H), range(nB), allowed)
        for h in range(H):
            S = torch.from_numpy(q[:, h] @ k[:, h].T * scale).masked_fill(~torch.from_numpy(mask), float("-inf"))
            p = torch.softmax(S, dim=-1).numpy()                         # library softmax
            p = np.nan_to_num(p)                                         # rows without keys: none here
            rect = np.add.reduceat(np.add.reduceat(p, edges, axis=0), edges, axis=1)
            for qb in range(nB):
                assert np.allclose(got[(h, qb)], rect[qb], atol=1e-12), (dense, h, qb)
                rows = min((qb + 1) * blk, N) - qb * blk
                assert abs(got[(h, qb)].sum() - rows) < 1e-9
                blk_allowed = mask[qb * blk:(qb + 1) * blk].reshape(-1, N).any(axis=0)
                for kb in range(nB):
                    if not blk_allowed[kb * blk:(kb + 1) * blk].any():
                        assert got[(h, qb)][kb] == 0.0
            if dense:
                ref = attention.block_mass(q, k, scale, blk, [h], range(nB))
                for qb in range(nB):
                    assert np.allclose(got[(h, qb)], ref[(h, qb)], atol=1e-12)
        # q == 0: uniform over each row's allowed keys
        got = attention.block_mass_restricted(np.zeros_like(q), k, scale, blk, [0], range(nB), allowed)
        for qb in range(nB):
            want = np.zeros(nB)
            for r in range(qb * blk, min((qb + 1) * blk, N)):
                keys = np.flatnonzero(mask[r])
                np.add.at(want, keys // blk, 1.0 / keys.size)
            assert np.allclose(got[(0, qb)], want, atol=1e-12)


# ----------------------------------------------------------------- LoSA ---
def read_losa_golden():
    cases = []
    with open(os.path.join(GOLDEN, "losa_select_cases.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            tau, masses, kept = [x.strip() for x in line.split("|")]
            cases.append((float(tau), [float(x) for x in masses.split()],
                          [int(x) for x in kept.split()]))
    return cases


def check_losa_golden(losa):
    for tau, masses, kept in read_losa_golden():
        got = list(losa.select_row(np.array(masses, dtype=np.float32), tau))
        assert got == kept, (tau, masses, got, kept)
        got = list(losa.select_row_fast(np.array(masses, dtype=np.float32), tau))
        assert got == kept, (tau, masses, got, kept)


def check_losa_bruteforce(losa, trials=300):
    """Enumerate every subset: the answer has minimum size among subsets whose
    quantised mass reaches the threshold, and is the top-k by (mass desc, id asc)."""
    rng = np.random.default_rng(13)
    for trial in range(trials):
        n = int(rng.integers(1, 9))
        if trial % 3 == 0:
            m = rng.choice([0.0, 0.125, 0.25, 0.5, 1.0], size=n)   # many ties
        else:
            m = rng.random(n) * rng.choice([1e-3, 1.0, 100.0])
        m = m.astype(np.float32)
        tau = float(rng.choice([0.3, 0.5, 0.9, 0.99, 1.0]))
        Q = [math.floor(Fraction(float(x)) * 2 ** 33) for x in m]   # exact rationals
        total = sum(Q)
        thr = math.ceil(tau * float(total))
        best = None
        for size in range(1, n + 1):
            for X in itertools.combinations(range(n), size):
                if sum(Q[i] for i in X) >= thr:
                    key = sorted((-Q[i], i) for i in X)
                    if best is None or key < best[0]:
                        best = (key, X)
            if best is not None:
                break
        want = sorted(best[1])
        assert list(losa.select_row(m, tau)) == want, (m, tau)
        assert list(losa.select_row_fast(m, tau)) == want, (m, tau)


def check_losa_properties(losa):
    rng = np.random.default_rng(17)
    for trial in range(50):
        n = int(rng.integers(2, 300))
        m = (rng.random(n) ** 8).astype(np.float32)
        kept = list(losa.select_row_fast(m, 0.99))
        mm = [Fraction(float(x)) for x in m]
        total = sum(mm)
        got = sum(mm[i] for i in kept)
        assert got >= Fraction(0.99) * total - Fraction(len(m), 2 ** 33)   # retained >= 99%
        # minimality: dropping the smallest kept block falls below the cut
        if len(kept) > 1:
            smallest = min(kept, key=lambda i: (mm[i], -i))
            assert got - mm[smallest] < Fraction(0.99) * total
        assert kept == sorted(kept)
