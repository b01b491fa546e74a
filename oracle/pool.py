"""Parallel evaluation of the attention oracle on the host cores (test and
benchmark infrastructure only: the CPU-baseline leg of bench.py).

No arithmetic of its own.  The query rows of a sample are split into tasks
(one head and the rows of one query frame each, since those rows share a key
set), and every task calls ``oracle.attention.attention_rows`` in a worker
process.  The workers read q, k, v (float64, exact copies of the bf16 inputs)
from memory-mapped files, so each head is held once in the page cache and
not copied per worker; each worker runs single-threaded numpy.

Workers are started with the ``spawn`` method (a process forked after the
parent has touched a GPU can hang), before the timed region.
"""
from __future__ import annotations

import multiprocessing as mp
import os
import shutil
import sys
import tempfile
import time
from typing import Dict, List, Sequence, Tuple

import numpy as np

_ARRAYS: Dict[str, np.ndarray] = {}


def _open(path: str) -> np.ndarray:
    a = _ARRAYS.get(path)
    if a is None:
        if len(_ARRAYS) >= 6:          # a new sample: drop the maps of the old files
            _ARRAYS.clear()
        a = np.load(path, mmap_mode="r")
        _ARRAYS[path] = a
    return a


def _task(args) -> Tuple[int, np.ndarray, np.ndarray, np.ndarray]:
    """One (head, row group): O and LSE of the rows from the oracle."""
    from oracle import attention as oatt
    tag, paths, rows, keys, scale = args
    q, k, v = (_open(p) for p in paths)
    O, L = oatt.attention_rows(q, k, v, scale, rows, [0], lambda _h, _r: keys, lambda _h, _r: 0)
    return tag, np.asarray(rows), O[0], L[0]


def _warm(_) -> int:
    return os.getpid()


class OraclePool:
    """A pool of single-threaded worker processes and a scratch folder for
    the memory-mapped inputs of one sample."""

    def __init__(self, workers: int = 0):
        self.workers = workers or len(os.sched_getaffinity(0))
        self.dir = tempfile.mkdtemp(prefix="bsa_oracle_")
        saved = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
        for k in saved:
            os.environ[k] = "1"
        # a spawned worker re-imports the parent's main script unless it is
        # hidden; the workers need only this module and numpy
        main = sys.modules.get("__main__")
        hidden = {a: getattr(main, a) for a in ("__file__", "__spec__") if main is not None and hasattr(main, a)}
        for a in hidden:
            setattr(main, a, None)
        try:
            self.pool = mp.get_context("spawn").Pool(self.workers)
        finally:
            for a, v in hidden.items():
                setattr(main, a, v)
            for k, v in saved.items():
                if v is None:
                    os.environ.pop(k, None)
                else:
                    os.environ[k] = v
        self.n = 0
        self.pool.map(_warm, range(4 * self.workers), chunksize=1)      # workers up before any timing

    def put_head(self, q: np.ndarray, k: np.ndarray, v: np.ndarray) -> Tuple[str, str, str]:
        """Write one head's q, k, v ([N, 1, d] float64) for the workers."""
        paths = []
        for name, a in (("q", q), ("k", k), ("v", v)):
            p = os.path.join(self.dir, f"{name}{self.n}.npy")
            np.save(p, np.ascontiguousarray(a, dtype=np.float64))
            paths.append(p)
        self.n += 1
        return tuple(paths)

    def drop_files(self):
        _ARRAYS.clear()
        for f in os.listdir(self.dir):
            os.unlink(os.path.join(self.dir, f))

    def attention_rows(self, heads: Sequence[Tuple[Tuple[str, str, str], np.ndarray]],
                       keys_of_row, group_of_row, scale: float):
        """Oracle O and LSE for every (head files, rows) pair; rows of one
        group (same key set) form one task.  Returns (list of (O, LSE) per
        head in the given row order, wall seconds of the parallel part)."""
        tasks = []
        for hi, (paths, rows) in enumerate(heads):
            groups: Dict[object, List[int]] = {}
            for r in np.asarray(rows).tolist():
                groups.setdefault(group_of_row(r), []).append(r)
            for g, rs in groups.items():
                tasks.append(((hi, g), paths, np.asarray(rs, dtype=np.int64), keys_of_row(rs[0]), scale))
        tasks.sort(key=lambda t: -len(t[2]) * len(t[3]))        # largest first
        t0 = time.perf_counter()
        parts = self.pool.map(_task, tasks, chunksize=1)
        dt = time.perf_counter() - t0
        out = []
        for hi, (_, rows) in enumerate(heads):
            rows = np.asarray(rows)
            pos = {int(r): i for i, r in enumerate(rows.tolist())}
            O = np.zeros((len(rows), 0))
            L = np.zeros(len(rows))
            for (h, _), rr, o, l in parts:
                if h != hi:
                    continue
                if O.shape[1] == 0:
                    O = np.zeros((len(rows), o.shape[1]))
                idx = np.array([pos[int(r)] for r in rr])
                O[idx] = o
                L[idx] = l
            out.append((O, L))
        return out, dt

    def close(self):
        self.pool.terminate()
        self.pool.join()
        shutil.rmtree(self.dir, ignore_errors=True)
