"""LVSA attended-frame sets (oracle; test infrastructure only).

Source: [LVSA] technical summary, section 2 "Method", core mechanism.  A
query frame t attends the frame set A(t) = G u W(t) instead of all frames
0..T-1, where G is the set of rotating global anchor frames and W(t) a local
temporal window that is widened where it overlaps anchors so that every
frame's budget |A(t)| stays at the target C (C = training horizon).

Readings taken where the page is open:
  * Anchors at step s: G_s = {f in [0, T) : (f - s) mod T_per == 0}, steps
    counted from 0.  The page fixes only the shift by s mod T_per and that
    every frame is an anchor exactly once over T_per consecutive steps.
  * Window and budget ("fill to budget"): A(t) = G_s u {t} plus the
    non-anchor frames nearest to t, taken in order of distance |f - t| and,
    at equal distance, the earlier frame (t - dist) first, until |A(t)| = C.
    The window is clipped at 0 and T-1; the growth continues on the open
    side.  The window size W then only has to be >= 1.
  * If |G_s u {t}| > C no set of size C holds every anchor and t; then
    A(t) = G_s u {t} and the call reports "over budget".  Anchors and t are
    never dropped.
  * The other reading, "fixed window" (attended_frames_window): the window
    holds W non-anchor frames, so |A(t)| = |G_s| + W and C plays no part.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np


def anchor_frames(T: int, T_per: int, s: int) -> List[int]:
    """G_s: frames f with (f - s) mod T_per == 0 ([LVSA] sec. 2, rotating anchors)."""
    return [f for f in range(T) if (f - s) % T_per == 0]


def attended_frames(T: int, T_per: int, W: int, C: int, s: int) -> Tuple[List[List[int]], bool]:
    """A(t) for every query frame t at step s, ascending; plus the over-budget flag.

    [LVSA] sec. 2: A(t) = G u W(t), window widened around anchors to keep
    |A(t)| = C.  Reading "fill to budget" (module docstring).
    """
    if T < 1 or T_per < 1 or W < 1 or C < 1 or s < 0:
        raise ValueError("T, T_per, W, C must be >= 1 and s >= 0")
    G = set(anchor_frames(T, T_per, s))
    out: List[List[int]] = []
    over = False
    for t in range(T):
        A = set(G)
        A.add(t)
        if len(A) > C:
            over = True
        need = C - len(A)
        dist = 1
        while need > 0 and (t - dist >= 0 or t + dist < T):
            for f in (t - dist, t + dist):          # earlier frame first at a tie
                if need > 0 and 0 <= f < T and f not in A:
                    A.add(f)
                    need -= 1
            dist += 1
        out.append(sorted(A))
    return out, over


def attended_frames_window(T: int, T_per: int, W: int, s: int) -> List[List[int]]:
    """A(t) under the fixed-window reading, ascending, for every query frame t.

    [LVSA] sec. 2: A(t) = G u W(t).  Reading "fixed window" (the other
    plain reading of the page, besides fill-to-budget): W(t) holds the W
    non-anchor frames nearest to t - t itself first when it is not an
    anchor, then by distance |f - t|, the earlier frame first at a tie - or
    every non-anchor frame when there are fewer than W.  Hence
    |A(t)| = |G_s| + min(W, T - |G_s|); t is always in A(t).
    """
    if T < 1 or T_per < 1 or W < 1 or s < 0:
        raise ValueError("T, T_per, W must be >= 1 and s >= 0")
    G = set(anchor_frames(T, T_per, s))
    free = [f for f in range(T) if f not in G]
    out: List[List[int]] = []
    for t in range(T):
        window = sorted(free, key=lambda f: (abs(f - t), f))[:W]
        out.append(sorted(G | {t} | set(window)))
    return out


def allowed_frames_matrix(A: List[List[int]], T: int) -> np.ndarray:
    """Boolean [T, T]: entry (t, f) is True iff f is in A(t)."""
    M = np.zeros((T, T), dtype=bool)
    for t, fr in enumerate(A):
        M[t, fr] = True
    return M


def token_frame(i, P: int):
    """Frame of token i when each frame holds P tokens: floor(i / P)."""
    return np.asarray(i) // P


def allowed_keys_for_row(q: int, A: List[List[int]], P: int, N: int) -> np.ndarray:
    """Key tokens query token q may attend: every token of every frame in A(frame(q)).

    [LVSA] sec. 2: the attention of query frame t is restricted to frames
    A(t); every token of an attended frame is visible (the cost per query is
    |A(t)| * P keys, sec. 2 complexity).
    """
    f = int(q) // P
    parts = [np.arange(g * P, min((g + 1) * P, N)) for g in A[f]]
    return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)


def dense_token_mask(A: List[List[int]], P: int, N: int) -> np.ndarray:
    """Explicit [N, N] boolean mask (small N only): mask[q, k] = frame(k) in A(frame(q))."""
    T = len(A)
    M = allowed_frames_matrix(A, T)
    fq = token_frame(np.arange(N), P)
    return M[fq[:, None], fq[None, :]]
