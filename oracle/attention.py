"""Masked softmax attention and LoSA block mass in float64 (oracle; test infrastructure only).

Definitions:
  * Attention of query token q of head h over its allowed keys K(q):
        s_k   = scale * <q_h, k_h>              (k in K(q))
        O[q]  = sum_k exp(s_k) v_k / sum_k exp(s_k)
        LSE[q] = log(sum_k exp(s_k))             (natural log)
    Bidirectional, no causal mask (the pages describe self-attention over the
    whole 3D token sequence of a video DiT: [LVSA] technical summary,
    section 1; [LoSA] section on the cost of video diffusion transformers).
    An empty K(q) gives O = 0 and LSE = -inf.
    LVSA restricts K(q) to the tokens of frames A(frame(q)) ([LVSA] sec. 2);
    LoSA restricts it to the kept key blocks of q's query block ([LoSA],
    section "Balancing efficiency and quality").  Both are exact masked
    attention, not an approximation of it.
  * LoSA block mass ([LoSA], same section: the dense measuring step records
    the exact attention mass between blocks): for head h, query block qb and
    key block kb,
        mass[h, qb, kb] = sum_{q in qb, q < N} sum_{k in kb, k < N} p_h(q, k)
    with p_h the dense softmax probabilities.

Inputs are the bf16 tensors converted exactly to float64.  Rows are computed
in groups with numpy matmuls (a library primitive) and no other reordering.
"""
from __future__ import annotations

from typing import Callable, Dict, Iterable, Sequence, Tuple

import numpy as np


def to_f64(x) -> np.ndarray:
    """Exact conversion of a bf16/fp32 torch tensor or array to float64 numpy."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu").to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


def attention_rows_with_keys(q: np.ndarray, k: np.ndarray, v: np.ndarray, h: int,
                             rows: np.ndarray, keys: np.ndarray, scale: float
                             ) -> Tuple[np.ndarray, np.ndarray]:
    """O [len(rows), d] and LSE [len(rows)] for query ``rows`` of head h over key set ``keys``.

    Direct evaluation of the definition in the module docstring; all rows
    share the same key set.
    """
    d = v.shape[2]
    if len(keys) == 0:
        return np.zeros((len(rows), d)), np.full(len(rows), -np.inf)
    S = (q[rows, h, :] @ k[keys, h, :].T) * scale           # [r, |K|]
    m = S.max(axis=1, keepdims=True)
    p = np.exp(S - m)
    l = p.sum(axis=1, keepdims=True)
    O = (p @ v[keys, h, :]) / l
    lse = (m + np.log(l))[:, 0]
    return O, lse


def attention_rows(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                   rows: Sequence[int], heads: Iterable[int],
                   keys_of_row: Callable[[int, int], np.ndarray],
                   group_of_row: Callable[[int, int], object] = None
                   ) -> Tuple[Dict[int, np.ndarray], Dict[int, np.ndarray]]:
    """Masked attention for selected rows and heads.

    ``keys_of_row(h, q)`` returns the allowed key tokens of row q in head h.
    ``group_of_row(h, q)`` (optional) returns a hashable key such that rows
    with equal keys have equal key sets; they are evaluated together.
    Returns dicts head -> O [len(rows), d] and head -> LSE [len(rows)].
    """
    rows = np.asarray(rows, dtype=np.int64)
    Os, Ls = {}, {}
    for h in heads:
        O = np.zeros((len(rows), v.shape[2]))
        L = np.zeros(len(rows))
        groups: Dict[object, list] = {}
        for i, r in enumerate(rows):
            g = group_of_row(h, int(r)) if group_of_row else ("row", int(r))
            groups.setdefault(g, []).append(i)
        for g, members in groups.items():
            members = np.asarray(members)
            keys = keys_of_row(h, int(rows[members[0]]))
            o, l = attention_rows_with_keys(q, k, v, h, rows[members], keys, scale)
            O[members] = o
            L[members] = l
        Os[h], Ls[h] = O, L
    return Os, Ls


def attention_dense_masked(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float,
                           mask: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Full O [N, H, d] and LSE [H, N] with an explicit [N, N] (or [H, N, N]) mask; small N only."""
    N, H, d = q.shape
    O = np.zeros((N, H, d))
    L = np.zeros((H, N))
    for h in range(H):
        mh = mask[h] if mask.ndim == 3 else mask
        S = (q[:, h, :] @ k[:, h, :].T) * scale
        S = np.where(mh, S, -np.inf)
        m = S.max(axis=1, keepdims=True)
        empty = ~np.isfinite(m[:, 0])
        m[empty] = 0.0
        p = np.exp(S - m)
        l = p.sum(axis=1, keepdims=True)
        with np.errstate(invalid="ignore", divide="ignore"):
            O[:, h, :] = np.where(empty[:, None], 0.0, (p @ v[:, h, :]) / l)
            L[h] = np.where(empty, -np.inf, (m + np.log(l))[:, 0])
    return O, L


def block_mass(q: np.ndarray, k: np.ndarray, scale: float, block: int,
               heads: Iterable[int], qblocks: Iterable[int]) -> Dict[Tuple[int, int], np.ndarray]:
    """mass[h, qb, :] (length ceil(N/block)) for the given heads and query blocks.

    [LoSA] "Balancing efficiency and quality": dense probabilities of the
    measuring step, summed over each (query block, key block) rectangle.
    """
    N = q.shape[0]
    nB = -(-N // block)
    out = {}
    for h in heads:
        for qb in qblocks:
            rows = np.arange(qb * block, min((qb + 1) * block, N))
            S = (q[rows, h, :] @ k[:, h, :].T) * scale            # [r, N]
            m = S.max(axis=1, keepdims=True)
            p = np.exp(S - m)
            p /= p.sum(axis=1, keepdims=True)
            mass = np.zeros(nB)
            for kb in range(nB):
                mass[kb] = p[:, kb * block:min((kb + 1) * block, N)].sum()
            out[(h, qb)] = mass
    return out


def block_mass_restricted(q: np.ndarray, k: np.ndarray, scale: float, block: int,
                          heads: Iterable[int], qblocks: Iterable[int],
                          allowed: Callable[[int, int], np.ndarray]) -> Dict[Tuple[int, int], np.ndarray]:
    """mass[h, qb, :] of attention restricted to allowed key sets.

    The LoSA measuring step ([LoSA] "Balancing efficiency and quality") run
    on attention that is already restricted, e.g. to LVSA's frames A(t)
    ([LVSA] sec. 2): p_h(q, k) is the softmax of q over allowed(h, q) only
    (zero elsewhere) and the mass of (qb, kb) sums it over the rectangle.
    Rows with no allowed key contribute nothing.
    """
    N = q.shape[0]
    nB = -(-N // block)
    out = {}
    for h in heads:
        for qb in qblocks:
            mass = np.zeros(nB)
            for r in range(qb * block, min((qb + 1) * block, N)):
                keys = np.asarray(allowed(h, r), dtype=np.int64)
                if keys.size == 0:
                    continue
                s = (k[keys, h, :] @ q[r, h, :]) * scale
                e = np.exp(s - s.max())
                e /= e.sum()
                np.add.at(mass, keys // block, e)
            out[(h, qb)] = mass
    return out


def block_mass_from_probabilities(p: np.ndarray, block: int) -> np.ndarray:
    """mass [nB, nB] from an explicit [N, N] probability matrix (brute force, small N)."""
    N = p.shape[0]
    nB = -(-N // block)
    mass = np.zeros((nB, nB))
    for qb in range(nB):
        for kb in range(nB):
            for qq in range(qb * block, min((qb + 1) * block, N)):
                mass[qb, kb] += p[qq, kb * block:min((kb + 1) * block, N)].sum()
    return mass
