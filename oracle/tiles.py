"""Query-tile -> key-tile lists on the 128-token grid (oracle; test infrastructure only).

Source: [LVSA] technical summary, section 2: LVSA is a block-sparse
attention pattern; query frame t attends frames A(t) and the cost is
|A(t)| * P * d per query (complexity paragraph).  A block-sparse kernel
visits, for each tile of 128 query rows, every 128-column key tile holding
at least one allowed (query, key) pair.

Definitions (element level, rows and columns restricted to [0, N)):
  * key tile kt is KEPT for query tile qt iff some q in qt, k in kt has
    frame(k) in A(frame(q));
  * a kept tile is PARTIAL iff some pair (q, k) with q in qt, k in kt, both
    < N, is not allowed, or the tile reaches past N (its last column >= N).

Because the frames of the rows of a tile form a contiguous range (and so do
the frames of its columns), the tests of "some pair" / "all pairs" reduce to
the same tests over the frame sub-matrix A[fq_lo..fq_hi, fk_lo..fk_hi];
this is what ``kept_tiles`` evaluates.  ``kept_tiles_bruteforce`` evaluates
the element-level definition directly and pins it on small inputs.
"""
from __future__ import annotations

import math
from typing import List, Tuple

import numpy as np

from .lvsa import allowed_frames_matrix, dense_token_mask

TILE = 128


def kept_tiles(A: List[List[int]], T: int, N: int, tile: int = TILE,
               qtiles=None) -> Tuple[List[List[int]], List[List[int]]]:
    """Per query tile: ascending kept key tiles and their partial flags (0/1).

    ``qtiles`` (optional) restricts the evaluation to those query tiles; the
    returned lists then follow that order.
    """
    if N % T:
        raise ValueError("N must be a multiple of T")
    P = N // T
    M = allowed_frames_matrix(A, T)
    nB = math.ceil(N / tile)
    idx: List[List[int]] = []
    flg: List[List[int]] = []
    for qt in (range(nB) if qtiles is None else qtiles):
        q_lo, q_hi = qt * tile, min((qt + 1) * tile, N) - 1
        fq_lo, fq_hi = q_lo // P, q_hi // P
        row_i, row_f = [], []
        for kt in range(nB):
            k_lo, k_hi = kt * tile, min((kt + 1) * tile, N) - 1
            fk_lo, fk_hi = k_lo // P, k_hi // P
            sub = M[fq_lo:fq_hi + 1, fk_lo:fk_hi + 1]
            if sub.any():
                row_i.append(kt)
                partial = (not sub.all()) or ((kt + 1) * tile > N)
                row_f.append(int(partial))
        idx.append(row_i)
        flg.append(row_f)
    return idx, flg


def kept_tiles_bruteforce(A: List[List[int]], T: int, N: int, tile: int = TILE):
    """Element-level evaluation of the definition (small N only)."""
    P = N // T
    mask = dense_token_mask(A, P, N)
    nB = math.ceil(N / tile)
    idx, flg = [], []
    for qt in range(nB):
        rows = slice(qt * tile, min((qt + 1) * tile, N))
        ri, rf = [], []
        for kt in range(nB):
            cols = slice(kt * tile, min((kt + 1) * tile, N))
            blk = mask[rows, cols]
            if blk.any():
                ri.append(kt)
                rf.append(int((not blk.all()) or (kt + 1) * tile > N))
        idx.append(ri)
        flg.append(rf)
    return idx, flg


def tile_pair_count(idx: List[List[int]]) -> int:
    """Number of kept (query tile, key tile) pairs."""
    return sum(len(r) for r in idx)


def exact_pair_count(A: List[List[int]], T: int, N: int) -> int:
    """Number of allowed (query, key) token pairs: sum over q of |A(frame(q))| * P."""
    P = N // T
    return sum(len(A[t]) * P * P for t in range(T))
