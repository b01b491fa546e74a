"""Seeded synthetic q/k/v generators, shared by the tests, the benchmark and
the oracle's callers.

This module holds none of the attention method's arithmetic: it only draws
random numbers and adds the input structure a workload asks for.

Recipe (one call per workload and step):
  * a ``torch.Generator`` on the target device seeded with ``seed``;
  * q, k, v drawn in that order as float32 N(0, 1), shape [N, H, d];
  * for workloads with temporal locality, ``amp * sinusoid(frame(i), d)`` is
    added to q and k (the same vector for every head), where token i belongs
    to frame floor(i / P) and sinusoid(f)[j] = sin(f * w_j) for j < d/2 and
    cos(f * w_{j-d/2}) otherwise, with w_j = 10000 ** (-2 j / d);
  * every tensor is rounded to bfloat16 (round to nearest even).

Per-step perturbation (LoSA reuse): x_s = x_0 + amp * eps_s with a fresh,
independent eps_s per step, drawn from the generator seeded ``seed + step``.
"""
from __future__ import annotations

import math

import torch


def frame_sinusoid(T: int, d: int, device="cpu") -> torch.Tensor:
    """[T, d] float32 table of the per-frame sinusoid described above."""
    half = d // 2
    j = torch.arange(half, dtype=torch.float64, device=device)
    w = torch.pow(torch.tensor(10000.0, dtype=torch.float64, device=device), -2.0 * j / d)
    f = torch.arange(T, dtype=torch.float64, device=device)[:, None]
    ang = f * w[None, :]
    return torch.cat([torch.sin(ang), torch.cos(ang)], dim=1).to(torch.float32)


def make_qkv(N: int, H: int, d: int, seed: int, device="cpu", T: int | None = None,
             locality: float = 0.0):
    """Return bf16 (q, k, v), each [N, H, d], drawn as described in the module doc."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    q = torch.randn((N, H, d), generator=g, dtype=torch.float32, device=device)
    k = torch.randn((N, H, d), generator=g, dtype=torch.float32, device=device)
    v = torch.randn((N, H, d), generator=g, dtype=torch.float32, device=device)
    if locality:
        assert T is not None and N % T == 0
        P = N // T
        e = frame_sinusoid(T, d, device=device)              # [T, d]
        add = (locality * e).repeat_interleave(P, dim=0)      # [N, d]
        q += add[:, None, :]
        k += add[:, None, :]
        del add
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def perturb(x: torch.Tensor, amp: float, seed: int) -> torch.Tensor:
    """bf16 x + amp * eps with eps ~ N(0,1) from a generator seeded ``seed``."""
    g = torch.Generator(device=x.device)
    g.manual_seed(int(seed))
    eps = torch.randn(x.shape, generator=g, dtype=torch.float32, device=x.device)
    return (x.to(torch.float32) + amp * eps).to(torch.bfloat16)


def workload_qkv(wl, step: int = 0, device="cpu"):
    """q, k, v for workload ``wl`` (a workloads.Workload) at denoising ``step``.

    LVSA workloads draw fresh inputs per step (seed = seed_base + step).
    LoSA workloads (perturb > 0) draw x_0 once from seed_base and perturb it
    at step s > 0 with seed seed_base + s.
    """
    if wl.perturb and step > 0:
        q, k, v = make_qkv(wl.N, wl.H, wl.d, wl.seed_base, device, wl.T, wl.locality)
        return (perturb(q, wl.perturb, wl.seed_base + 100000 + 3 * step),
                perturb(k, wl.perturb, wl.seed_base + 100001 + 3 * step),
                perturb(v, wl.perturb, wl.seed_base + 100002 + 3 * step))
    return make_qkv(wl.N, wl.H, wl.d, wl.seed_base + step, device, wl.T, wl.locality)


def sample_rows(N: int, P: int, n: int, seed: int, block: int = 128):
    """Seeded, stratified sample of query rows for full-size spot checks.

    Always includes the first and last rows, rows on both sides of frame
    boundaries and of 128-row tile boundaries, and the last partial tile;
    the rest are uniform.  Returns a sorted int64 tensor of unique rows.
    """
    g = torch.Generator()
    g.manual_seed(int(seed))
    T = N // P
    rows = {0, N - 1, max(0, N - (N % block or block)), N - 2 if N > 1 else 0}
    nb = max(1, n // 8)
    for f in torch.randint(1, max(2, T), (nb,), generator=g).tolist():
        b = f * P
        rows.update({max(0, b - 1), min(N - 1, b)})
    for t in torch.randint(1, max(2, math.ceil(N / block)), (nb,), generator=g).tolist():
        b = t * block
        rows.update({max(0, b - 1), min(N - 1, b)})
    while len(rows) < n:
        rows.add(int(torch.randint(0, N, (1,), generator=g)))
    return torch.tensor(sorted(rows), dtype=torch.int64)
