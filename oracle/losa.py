"""LoSA minimal 99%-mass key-block selection (oracle; test infrastructure only).

Source: [LoSA] section "LoSA's innovative approach" (keep 99% of the
attention mass; attention weight concentrates in few blocks) and section
"Balancing efficiency and quality" (per attention head and query block, the
minimal set of key/value blocks needed to hold 99% of the mass is found once
and frozen for every later denoising step).

The algorithm, step by step, per (head, query block) row of block masses:
  1. quantise each mass to an integer, Q_kb = floor(mass_kb * 2**33)
     (exact: float32 -> float64 -> scale by a power of two -> floor);
  2. order the key blocks by Q descending, equal Q by key-block id ascending;
  3. total = sum of Q;  threshold = ceil(tau * total) with one IEEE float64
     multiply (tau * float64(total)), and never more than the total (a row
     total above 2**53 can round up when converted to float64; the kept set
     holds at least the fraction tau, so it needs at most the whole row);
  4. keep the shortest prefix of the order whose running sum of Q reaches the
     threshold (at least one block);
  5. emit the kept key-block ids in ascending order.

Readings: "minimal set" is the greedy largest-first prefix, which has the
fewest blocks of any set holding the threshold when masses are >= 0; ties
between equal masses go to the lower block id; the integer quantisation
makes the cut independent of summation order.  Masses must be finite,
>= 0 and < 2**14; a row has at most 65536 blocks.
"""
from __future__ import annotations

import math
from typing import List, Tuple

import numpy as np

QSHIFT = 33


def quantise(mass_row) -> List[int]:
    """Step 1: Q_kb = floor(mass_kb * 2**33) as exact Python integers."""
    out = []
    for m in np.asarray(mass_row, dtype=np.float32).tolist():
        m = float(m)                       # float32 value, exact in float64
        if not (m >= 0.0 and m < 2.0 ** 14):
            raise ValueError("block mass must be finite, >= 0 and < 2**14")
        out.append(math.floor(math.ldexp(m, QSHIFT)))
    return out


def select_row(mass_row, tau: float) -> List[int]:
    """Steps 1-5 for one row; returns the kept key-block ids ascending."""
    if not (0.0 < tau <= 1.0):
        raise ValueError("tau must be in (0, 1]")
    Q = quantise(mass_row)
    n = len(Q)
    if n == 0:
        return []
    order = sorted(range(n), key=lambda kb: (-Q[kb], kb))
    total = sum(Q)
    threshold = min(math.ceil(tau * float(total)), total)
    running = 0
    k = n
    for i, kb in enumerate(order):
        running += Q[kb]
        if running >= threshold:
            k = i + 1
            break
    return sorted(order[:k])


def select(mass, tau: float) -> Tuple[np.ndarray, np.ndarray]:
    """Whole tensor: mass [H, nQB, nKB] float32 -> idx [H, nQB, nKB] int32 (padded -1), cnt [H, nQB] int32."""
    mass = np.asarray(mass, dtype=np.float32)
    H, nQB, nKB = mass.shape
    idx = np.full((H, nQB, nKB), -1, dtype=np.int32)
    cnt = np.zeros((H, nQB), dtype=np.int32)
    for h in range(H):
        for qb in range(nQB):
            kept = select_row_fast(mass[h, qb], tau)
            idx[h, qb, :len(kept)] = kept
            cnt[h, qb] = len(kept)
    return idx, cnt


def select_row_fast(mass_row, tau: float) -> np.ndarray:
    """Same steps as ``select_row`` with numpy int64 arrays (used for large tensors).

    Exactness: Q < 2**47 per entry and the row total stays below 2**63, so
    the int64 running sums are exact; the threshold is the same float64
    product as in ``select_row``.
    """
    if not (0.0 < tau <= 1.0):
        raise ValueError("tau must be in (0, 1]")
    m = np.asarray(mass_row, dtype=np.float32).astype(np.float64)
    if m.size == 0:
        return np.zeros(0, dtype=np.int32)
    if not (np.all(m >= 0.0) and np.all(m < 2.0 ** 14)):
        raise ValueError("block mass must be finite, >= 0 and < 2**14")
    Q = np.floor(np.ldexp(m, QSHIFT)).astype(np.int64)
    kb = np.arange(m.size)
    order = np.lexsort((kb, -Q))                 # Q desc, then kb asc
    run = np.cumsum(Q[order])
    total = int(run[-1])
    threshold = min(math.ceil(tau * float(total)), total)
    k = int(np.argmax(run >= threshold)) + 1
    return np.sort(order[:k]).astype(np.int32)
