"""Helpers for the GPU parity tests: run the CUDA path through the C ABI,
run the oracle on the same inputs (copied to the host), compare.

Tolerances (attention outputs, bf16 in / fp32 accumulate):
  O:    max |gpu - oracle| <= 1e-2 and mean |gpu - oracle| <= 1e-3
  LSE:  max |gpu - oracle| <= 1e-3  (fp32 scores and sums: ~1e-5 expected;
        the bound leaves room for the approximate exp2 and log2)
  mass: max |gpu - oracle| / rows(qb) <= 1e-4 (normalised block mass)
Index lists and selections: bit-exact.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from oracle import attention as oatt
from oracle import lvsa as olvsa

O_MAX, O_MEAN, LSE_MAX, MASS_MAX = 1e-2, 1e-3, 1e-3, 1e-4


def need_gpu():
    if not torch.cuda.is_available():
        raise RuntimeError("GPU test run without a CUDA device")


def head_f64(x: torch.Tensor, h: int) -> np.ndarray:
    """[N, 1, d] float64 numpy copy of head h of a bf16 CUDA tensor (exact)."""
    return x[:, h:h + 1, :].to("cpu").to(torch.float64).numpy()


def oracle_rows(q, k, v, scale, rows, heads, keys_of_row, group_of_row):
    """Oracle O [len(rows), d] and LSE [len(rows)] per head, one head at a time."""
    Os, Ls = {}, {}
    for h in heads:
        qh, kh, vh = head_f64(q, h), head_f64(k, h), head_f64(v, h)
        O, L = oatt.attention_rows(qh, kh, vh, scale, rows, [0],
                                   lambda _h, r: keys_of_row(h, r),
                                   (lambda _h, r: group_of_row(h, r)) if group_of_row else None)
        Os[h], Ls[h] = O[0], L[0]
    return Os, Ls


def compare_rows(o_gpu, lse_gpu, Os, Ls, rows, what=""):
    rows_t = torch.as_tensor(np.asarray(rows), dtype=torch.long, device=o_gpu.device)
    errs, maxe = [], 0.0
    for h in Os:
        og = o_gpu[rows_t, h, :].to(torch.float64).cpu().numpy()
        lg = lse_gpu[h, rows_t].to(torch.float64).cpu().numpy()
        e = np.abs(og - Os[h])
        errs.append(e.ravel())
        maxe = max(maxe, float(e.max()))
        lo = Ls[h]
        fin = np.isfinite(lo)
        assert np.array_equal(fin, np.isfinite(lg)), f"{what} h={h}: LSE finiteness differs"
        if fin.any():
            le = float(np.abs(lg[fin] - lo[fin]).max())
            assert le <= LSE_MAX, f"{what} h={h}: LSE max err {le}"
    mean = float(np.concatenate(errs).mean())
    assert maxe <= O_MAX, f"{what}: O max err {maxe}"
    assert mean <= O_MEAN, f"{what}: O mean err {mean}"
    return maxe, mean


def lvsa_keys(A, P, N):
    return (lambda h, r: olvsa.allowed_keys_for_row(r, A, P, N)), (lambda h, r: r // P)


def block_keys(idx_np, cnt_np, N, block=128):
    def keys(h, r):
        qb = r // block
        kept = idx_np[h, qb, :cnt_np[h, qb]]
        parts = [np.arange(kb * block, min((kb + 1) * block, N)) for kb in kept if 0 <= kb]
        return np.concatenate(parts) if parts else np.zeros(0, dtype=np.int64)
    return keys, (lambda h, r: r // block)


def dense_keys(N):
    allk = np.arange(N)
    return (lambda h, r: allk), (lambda h, r: 0)
