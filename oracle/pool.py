"""Timing the oracle on the host cores: independent solves spread over a process pool.

Test and baseline infrastructure, like the rest of `oracle/`: it runs the plain binary64
solver (oracle/solver.py) as it stands, one task per matrix or column strip, and reports
the work done and the time taken. Column strips are a valid sample of a solve because
every step couples only the columns of one block (r) or the rows of one column (c).

    python -m oracle.pool <tasks.npz> <workers>

reads the task matrices W_0, W_1, ... and a JSON list `meta` of (kind, group, iters, amax,
update) from the .npz file, solves them on a pool of `workers` spawned processes (the pool
is started and warmed before the clock starts) and prints one JSON object:
{"work": sum of elements x iterations, "wall_s": ..., "cpu_s": summed per-task seconds,
 "workers": ..., "tasks": ...}.
"""
from __future__ import annotations

import json
import multiprocessing as mp
import sys
import time

import numpy as np


def solve_task(task):
    """(W binary64, kind, group, iters, amax or None, update) -> (elements x iters, seconds)."""
    from oracle import formats as F
    from oracle import solver as S
    W, kind, group, iters, amax, update = task
    t0 = time.perf_counter()
    S.solve(W, F.make_format(kind, group), iters, amax=amax, update=update)
    return W.size * iters, time.perf_counter() - t0


def _ready(_):
    import oracle.solver  # noqa: F401  (import cost paid before the clock starts)
    return 0


def run(tasks, workers: int) -> dict:
    workers = max(1, min(int(workers), len(tasks)))
    if workers == 1:
        _ready(0)
        t0 = time.perf_counter()
        res = [solve_task(t) for t in tasks]
        wall = time.perf_counter() - t0
    else:
        with mp.get_context("spawn").Pool(workers) as pool:
            pool.map(_ready, range(workers), chunksize=1)
            t0 = time.perf_counter()
            res = pool.map(solve_task, tasks, chunksize=1)
            wall = time.perf_counter() - t0
    return {"work": int(sum(r[0] for r in res)), "wall_s": wall,
            "cpu_s": float(sum(r[1] for r in res)), "workers": workers, "tasks": len(tasks)}


def save_tasks(path: str, tasks) -> None:
    arrays = {"W_%d" % i: np.ascontiguousarray(t[0], dtype=np.float64)
              for i, t in enumerate(tasks)}
    meta = [[t[1], int(t[2]), int(t[3]), None if t[4] is None else float(t[4]), t[5]]
            for t in tasks]
    np.savez(path, meta=np.array(json.dumps(meta)), **arrays)


def load_tasks(path: str):
    d = np.load(path)
    meta = json.loads(str(d["meta"]))
    return [(d["W_%d" % i], m[0], m[1], m[2], m[3], m[4]) for i, m in enumerate(meta)]


if __name__ == "__main__":
    print(json.dumps(run(load_tasks(sys.argv[1]), int(sys.argv[2]))), flush=True)
