"""Planted mistakes in the oracle must be caught by the pins (CPU only).

Each case copies an oracle module, plants one plausible mistake (a sign, a
tie-break, a transposed operand, a dropped term), and checks that at least
one pin fails.  This shows the pins constrain the oracle rather than echo it.
"""
import math
import types

import numpy as np
import pytest

from oracle import attention, losa, lvsa, tiles
from tests import pins


def clone(mod):
    m = types.ModuleType(mod.__name__ + "_mutant")
    m.__dict__.update({k: v for k, v in mod.__dict__.items() if not k.startswith("__")})
    return m


def fails(check, *mods):
    try:
        check(*mods)
    except AssertionError:
        return True
    return False


def mutant_lvsa_anchor_sign():
    m = clone(lvsa)
    m.anchor_frames = lambda T, T_per, s: [f for f in range(T) if (f + s) % T_per == 0]

    def attended(T, T_per, W, C, s, _orig=lvsa.attended_frames):
        # re-run the original fill with the mutated anchors
        G = set(m.anchor_frames(T, T_per, s))
        out, over = [], False
        for t in range(T):
            A = set(G) | {t}
            over |= len(A) > C
            need, dist = C - len(A), 1
            while need > 0 and (t - dist >= 0 or t + dist < T):
                for f in (t - dist, t + dist):
                    if need > 0 and 0 <= f < T and f not in A:
                        A.add(f); need -= 1
                dist += 1
            out.append(sorted(A))
        return out, over
    m.attended_frames = attended
    return m


def mutant_lvsa_tiebreak():
    m = clone(lvsa)

    def attended(T, T_per, W, C, s):
        G = set(lvsa.anchor_frames(T, T_per, s))
        out, over = [], False
        for t in range(T):
            A = set(G) | {t}
            over |= len(A) > C
            need, dist = C - len(A), 1
            while need > 0 and (t - dist >= 0 or t + dist < T):
                for f in (t + dist, t - dist):            # later frame first: wrong
                    if need > 0 and 0 <= f < T and f not in A:
                        A.add(f); need -= 1
                dist += 1
            out.append(sorted(A))
        return out, over
    m.attended_frames = attended
    return m


def test_lvsa_sign_caught():
    assert fails(pins.check_lvsa_golden, mutant_lvsa_anchor_sign())


def test_lvsa_tiebreak_caught():
    m = mutant_lvsa_tiebreak()
    assert fails(pins.check_lvsa_golden, m)
    assert fails(pins.check_lvsa_bruteforce, m)


def mutant_lvsa_window(kind):
    """Fixed-window reading with one planted mistake."""
    m = clone(lvsa)

    def window(T, T_per, W, s):
        G = set(lvsa.anchor_frames(T, T_per, s))
        free = [f for f in range(T) if f not in G]
        out = []
        for t in range(T):
            if kind == "tie":            # later frame first at equal distance
                order = sorted(free, key=lambda f: (abs(f - t), -f))
            else:
                order = sorted(free, key=lambda f: (abs(f - t), f))
            if kind == "no_t":           # t not counted in its own window
                order = [f for f in order if f != t]
            n = W - 1 if kind == "short" else W
            out.append(sorted(G | {t} | set(order[:n])))
        return out
    m.attended_frames_window = window
    return m


@pytest.mark.parametrize("kind", ["tie", "no_t", "short"])
def test_lvsa_window_mistakes_caught(kind):
    m = mutant_lvsa_window(kind)
    assert fails(pins.check_lvsa_window_golden, m)
    assert fails(pins.check_lvsa_window_bruteforce, m)


def test_restricted_mass_normaliser_caught():
    m = clone(attention)

    def restricted(q, k, scale, block, heads, qblocks, allowed):
        N = q.shape[0]
        nB = -(-N // block)
        out = {}
        for h in heads:
            for qb in qblocks:
                mass = np.zeros(nB)
                for r in range(qb * block, min((qb + 1) * block, N)):
                    keys = np.asarray(allowed(h, r), dtype=np.int64)
                    s_all = (k[:, h, :] @ q[r, h, :]) * scale
                    e = np.exp(s_all - s_all.max())
                    e /= e.sum()                          # normalised over every key: wrong
                    np.add.at(mass, keys // block, e[keys])
                out[(h, qb)] = mass
        return out
    m.block_mass_restricted = restricted
    assert fails(pins.check_block_mass_restricted, m, lvsa)


def test_tiles_partial_flag_caught():
    m = clone(tiles)

    def kept(A, T, N, tile=128):
        idx, flg = tiles.kept_tiles(A, T, N, tile)
        # forgets the "reaches past N" condition
        P = N // T
        M = lvsa.allowed_frames_matrix(A, T)
        out = []
        for qt, (ri, rf) in enumerate(zip(idx, flg)):
            q_lo, q_hi = qt * tile, min((qt + 1) * tile, N) - 1
            row = []
            for kt in ri:
                k_lo, k_hi = kt * tile, min((kt + 1) * tile, N) - 1
                sub = M[q_lo // P:q_hi // P + 1, k_lo // P:k_hi // P + 1]
                row.append(int(not sub.all()))
            out.append(row)
        return idx, out
    m.kept_tiles = kept
    assert fails(pins.check_tiles_vs_bruteforce, m, lvsa)


def test_attention_transposed_operand_caught():
    m = clone(attention)

    def dense(q, k, v, scale, mask):
        return attention.attention_dense_masked(q, k, k, scale, mask)   # k used as v
    m.attention_dense_masked = dense
    assert fails(pins.check_attention_closed_forms, m, lvsa)


def test_attention_dropped_scale_caught():
    m = clone(attention)

    def dense(q, k, v, scale, mask):
        return attention.attention_dense_masked(q, k, v, 1.0, mask)    # scale dropped
    m.attention_dense_masked = dense
    assert fails(pins.check_attention_vs_sdpa, m, lvsa)


def test_block_mass_unnormalised_caught():
    m = clone(attention)

    def bm(q, k, scale, block, heads, qblocks):
        N = q.shape[0]
        nB = -(-N // block)
        out = {}
        for h in heads:
            for qb in qblocks:
                rows = np.arange(qb * block, min((qb + 1) * block, N))
                S = (q[rows, h] @ k[:, h].T) * scale
                p = np.exp(S - S.max(axis=1, keepdims=True))        # not normalised
                out[(h, qb)] = np.array([p[:, kb * block:(kb + 1) * block].sum() for kb in range(nB)])
        return out
    m.block_mass = bm
    assert fails(pins.check_block_mass, m)


def test_losa_tiebreak_caught():
    m = clone(losa)

    def sel(mass_row, tau):
        Q = losa.quantise(mass_row)
        order = sorted(range(len(Q)), key=lambda kb: (-Q[kb], -kb))   # higher id first: wrong
        thr = math.ceil(tau * float(sum(Q)))
        run = 0
        for i, kb in enumerate(order):
            run += Q[kb]
            if run >= thr:
                return sorted(order[:i + 1])
        return sorted(order)
    m.select_row = sel
    m.select_row_fast = sel
    assert fails(pins.check_losa_golden, m)


def test_losa_threshold_floor_caught():
    m = clone(losa)

    def sel(mass_row, tau):
        Q = losa.quantise(mass_row)
        order = sorted(range(len(Q)), key=lambda kb: (-Q[kb], kb))
        thr = math.floor(tau * float(sum(Q))) - 2 ** 31      # threshold too low
        run = 0
        for i, kb in enumerate(order):
            run += Q[kb]
            if run >= thr:
                return sorted(order[:i + 1])
        return sorted(order)
    m.select_row = sel
    m.select_row_fast = sel
    assert fails(pins.check_losa_golden, m) or fails(pins.check_losa_bruteforce, m)
