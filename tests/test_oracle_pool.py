"""The oracle's multiprocess runner (used only by bench.py's CPU-baseline
leg) returns exactly what the oracle returns when called directly: it splits
rows into tasks and adds no arithmetic."""
import numpy as np
import pytest
import torch

from oracle import attention as oatt
from oracle import lvsa as olvsa
from oracle.pool import OraclePool
from block_sparse_attention_lvsa_b200 import inputs
from block_sparse_attention_lvsa_b200.workloads import WORKLOADS


@pytest.mark.timeout(300)
def test_pool_equals_direct_oracle():
    wl = WORKLOADS["tiny"]
    q, k, v = inputs.workload_qkv(wl, 1, device="cpu")
    A, _ = olvsa.attended_frames(wl.T, wl.T_per, wl.W, wl.C, 1)
    keys = lambda r: olvsa.allowed_keys_for_row(r, A, wl.P, wl.N)      # noqa: E731
    rows = inputs.sample_rows(wl.N, wl.P, 100, 3).numpy()
    pool = OraclePool(workers=3)
    try:
        work = []
        for h in range(wl.H):
            qh, kh, vh = (x[:, h:h + 1, :].to(torch.float64).numpy() for x in (q, k, v))
            work.append((pool.put_head(qh, kh, vh), rows))
        out, dt = pool.attention_rows(work, keys, lambda r: r // wl.P, wl.scale)
        assert dt > 0
    finally:
        pool.close()
    for h in range(wl.H):
        qh, kh, vh = (x[:, h:h + 1, :].to(torch.float64).numpy() for x in (q, k, v))
        O, L = oatt.attention_rows(qh, kh, vh, wl.scale, rows, [0], lambda _h, r: keys(r), lambda _h, r: r // wl.P)
        assert np.array_equal(out[h][0], O[0])
        assert np.array_equal(out[h][1], L[0])
