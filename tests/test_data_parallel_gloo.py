"""Data-parallel path on CPU: two gloo ranks, each with a contiguous frame shard.

Each rank computes its shard's forward, data gradient and weight/bias gradients with the
oracle (frames are independent, so a shard is a problem of its own once its indices are
rebased), sums dW/db with the same all-reduce helper the multi-GPU bench uses, and the
results must equal the whole batch's: outputs row for row, gradients up to the order of
the fp64 sums.
"""
import datetime
import os
import socket

import numpy as np
import pytest

from sparse_convolution_pruned_b200 import workloads as wl
from sparse_convolution_pruned_b200.data_parallel import shard_frames

WORLD = 2


def _workload():
    return wl.custom_conv(seed=61, T=7, H=6, W=9, keep_frac=[0.5, 0.2, 1.0, 0.0, 0.4, 0.6, 0.3], Cin=8, Cout=5,
                          dtype="f32")


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from sparse_convolution_pruned_b200.data_parallel import allreduce_grads

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        w = _workload()
        sh = shard_frames(w.coords, w.frame_off, rank, world)
        nbr, _, st = oracle.build_index(sh.coords, sh.frame_off, sh.T, w.H, w.W, want_map=False)
        X, dY = w.X[sh.r0:sh.r1], w.dY[sh.r0:sh.r1]
        Y = oracle.fwd(X, nbr, w.Wt, w.bias)
        dX = oracle.bwd_data(dY, nbr, w.Wt)
        dW, db = oracle.bwd_weight(dY, X, nbr)
        grads = torch.from_numpy(np.concatenate([dW.ravel(), db.ravel()]).astype(np.float64))
        allreduce_grads(grads)
        q.put((rank, sh.r0, sh.r1, int(st), Y, dX, grads.numpy()))
    finally:
        dist.destroy_process_group()


def test_shards_cover_the_batch_exactly():
    w = _workload()
    rows, frames = [], []
    for r in range(3):
        sh = shard_frames(w.coords, w.frame_off, r, 3)
        assert sh.frame_off[0] == 0 and sh.frame_off[-1] == sh.n
        assert (sh.coords[:, 0] >= 0).all() and (sh.coords[:, 0] < max(sh.T, 1)).all()
        rows.append((sh.r0, sh.r1))
        frames.append((sh.f0, sh.f1))
    assert rows[0][0] == 0 and rows[-1][1] == w.n
    assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
    assert frames[0][0] == 0 and frames[-1][1] == w.T
    with pytest.raises(ValueError):
        shard_frames(w.coords, w.frame_off, 2, 2)


def test_two_gloo_ranks_match_the_whole_batch(orc):
    import torch.multiprocessing as mp

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, WORLD, port, q)) for r in range(WORLD)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(WORLD)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    res.sort(key=lambda t: t[0])

    w = _workload()
    nbr, _, st = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    assert st == 0
    Y = orc.fwd(w.X, nbr, w.Wt, w.bias)
    dX = orc.bwd_data(w.dY, nbr, w.Wt)
    dW, db = orc.bwd_weight(w.dY, w.X, nbr)
    full = np.concatenate([dW.ravel(), db.ravel()])
    for rank, r0, r1, sst, Ys, dXs, grads in res:
        assert sst == 0
        np.testing.assert_array_equal(Ys, Y[r0:r1])     # same per-token sums, same order
        np.testing.assert_array_equal(dXs, dX[r0:r1])
        np.testing.assert_allclose(grads, full, rtol=1e-12, atol=1e-12)
    assert res[0][2] == res[1][1] and res[-1][2] == w.n
