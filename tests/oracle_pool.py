"""Frame-parallel runs of the oracle for full-size parity checks (test infrastructure).

Neighbours never cross frames, so every output row of the convolution, of its data
gradient and of the adapter depends only on rows of its own frame.  The oracle's
single-threaded functions are therefore run unchanged on contiguous frame ranges in
separate processes (each range with its neighbour table rebased to the range) and the
rows are put back in place: those rows are exactly the oracle's.  The weight and bias
gradients are sums over tokens; each range's partial sum is the oracle's fp64 result
for that range and the parent adds them (fp64, so the reference moves by rounding only).

Workers are started with 'spawn': the parent holds a CUDA context, and a process forked
from it could hang.
"""
from __future__ import annotations

import multiprocessing as mp
import os

import numpy as np


def frame_ranges(frame_off, parts):
    """Split frames into at most `parts` contiguous ranges of about equal token counts."""
    T = len(frame_off) - 1
    n = int(frame_off[-1])
    cuts = [0]
    for p in range(1, parts):
        f = int(np.searchsorted(frame_off, n * p / parts, side="left"))
        f = min(max(f, cuts[-1]), T)
        if f > cuts[-1]:
            cuts.append(f)
    if cuts[-1] != T:
        cuts.append(T)
    return [(cuts[i], cuts[i + 1]) for i in range(len(cuts) - 1)]


def _rebase(nbr, r0, r1):
    sub = nbr[r0:r1]
    return np.where(sub >= 0, sub - r0, -1).astype(np.int32)


def _conv_task(task):
    import oracle
    X, dY, sub_n, Wt, bias, do_fwd, do_bwd = task
    out = {}
    if do_fwd:
        out["Y"] = oracle.fwd(X, sub_n, Wt, bias)
    if do_bwd:
        out["dX"] = oracle.bwd_data(dY, sub_n, Wt)
        out["dW"], out["db"] = oracle.bwd_weight(dY, X, sub_n)
    return out


def _adapter_task(task):
    import oracle
    X, sub_n, Wd, Wc, Wu = task
    return oracle.adapter_fwd(X, sub_n, 0, X.shape[0], Wd, Wc, Wu)


def _down_task(task):
    import oracle
    X, Wd = task
    return oracle.down_proj(X, Wd)


def _workers():
    return max(1, min(32, os.cpu_count() or 1))


def conv_full(w, nbr, do_fwd=True, do_bwd=True):
    """Oracle Y (n x Cout), dX (n x Cin), dW, db of a whole conv workload, in parallel."""
    workers = _workers()
    rngs = frame_ranges(w.frame_off, 4 * workers)
    tasks = []
    for f0, f1 in rngs:
        r0, r1 = int(w.frame_off[f0]), int(w.frame_off[f1])
        tasks.append((w.X[r0:r1], w.dY[r0:r1] if do_bwd else None, _rebase(nbr, r0, r1), w.Wt, w.bias,
                      do_fwd, do_bwd))
    with mp.get_context("spawn").Pool(workers) as pool:
        parts = pool.map(_conv_task, tasks, chunksize=1)
    res = {}
    if do_fwd:
        res["Y"] = np.concatenate([p["Y"] for p in parts], 0)
    if do_bwd:
        res["dX"] = np.concatenate([p["dX"] for p in parts], 0)
        res["dW"] = np.sum([p["dW"] for p in parts], axis=0)
        res["db"] = np.sum([p["db"] for p in parts], axis=0)
    return res


def adapter_full(a, nbr):
    """Oracle adapter output (n x D) of a whole long-video workload, in parallel."""
    workers = _workers()
    rngs = frame_ranges(a.frame_off, 4 * workers)
    tasks = []
    for f0, f1 in rngs:
        r0, r1 = int(a.frame_off[f0]), int(a.frame_off[f1])
        tasks.append((a.X[r0:r1], _rebase(nbr, r0, r1), a.Wd, a.Wc, a.Wu))
    with mp.get_context("spawn").Pool(workers) as pool:
        parts = pool.map(_adapter_task, tasks, chunksize=1)
    return np.concatenate(parts, 0)


def down_proj_full(X, Wd):
    """Oracle down-projection bf16(X Wd^T) of every row, rows split over worker processes
    (each row is independent)."""
    workers = _workers()
    n = X.shape[0]
    cuts = np.linspace(0, n, 4 * workers + 1).astype(np.int64)
    tasks = [(X[a:b], Wd) for a, b in zip(cuts[:-1], cuts[1:]) if b > a]
    with mp.get_context("spawn").Pool(workers) as pool:
        parts = pool.map(_down_task, tasks, chunksize=1)
    return np.concatenate(parts, 0)
