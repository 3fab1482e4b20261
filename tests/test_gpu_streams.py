"""svconv_bwd from several host threads and streams, one of them capturing a CUDA graph.

At 64 channels svconv_bwd forks a side stream of the library off the caller's
stream.  Each (device, caller stream) pair has its own side stream, so a capture
on one stream must neither pull in nor wait on another thread's eager calls on
another stream, and a capture on a stream that has no side stream yet must still
give the same gradients (the two launches then run in order on the caller's
stream).  Every result is compared bit for bit with a plain call on one stream.
"""
import threading

import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_convolution_pruned_b200 import build, svconv
    build.build()
    return svconv


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(dtype) if dtype is not None else t).cuda()


class Bufs:
    def __init__(self, sv, w):
        self.dX = torch.empty((w.n, w.Cin), dtype=torch.bfloat16, device="cuda")
        self.dW = torch.empty((w.Cout, 9, w.Cin), device="cuda")
        self.db = torch.empty((w.Cout,), device="cuda")
        need = sv.svconv_bwd_workspace_size(sv.BF16, w.n, w.Cin, w.Cout)
        self.ws = torch.empty((max(16, need),), dtype=torch.uint8, device="cuda")

    def run(self, sv, dY, X, nbr, Wt, stream):
        sv.svconv_bwd(dY, X, nbr, Wt, dX=self.dX, dW=self.dW, db=self.db, workspace=self.ws, stream=stream)

    def equal(self, ref):
        return torch.equal(self.dX, ref.dX) and torch.equal(self.dW, ref.dW) and torch.equal(self.db, ref.db)


def test_bwd_two_threads_one_capturing(sv):
    w = wl.small_c_bf16()
    nbr, _ = sv.svconv_build_index(_dev(w.coords), _dev(w.frame_off), w.T, w.H, w.W)
    X, Wt, dY = _dev(w.X, torch.bfloat16), _dev(w.Wt, torch.bfloat16), _dev(w.dY, torch.bfloat16)
    ref = Bufs(sv, w)
    ref.run(sv, dY, X, nbr, Wt, torch.cuda.current_stream())
    torch.cuda.synchronize()

    s1, s2, s3 = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    a, b, c = Bufs(sv, w), Bufs(sv, w), Bufs(sv, w)
    # first calls on s1 and s2 outside capture: their side streams are created here
    for bufs, s in ((a, s1), (b, s2)):
        with torch.cuda.stream(s):
            bufs.run(sv, dY, X, nbr, Wt, s)
    torch.cuda.synchronize()
    for bufs in (a, b):
        bufs.dX.zero_(), bufs.dW.zero_(), bufs.db.zero_()
    torch.cuda.synchronize()

    start = threading.Barrier(2)
    errors = []
    g = torch.cuda.CUDAGraph()

    def capture():
        try:
            start.wait()
            with torch.cuda.graph(g, stream=s1, capture_error_mode="thread_local"):
                for _ in range(3):
                    a.run(sv, dY, X, nbr, Wt, s1)
        except Exception as e:  # pragma: no cover - reported below
            errors.append(e)

    def eager():
        try:
            start.wait()
            for _ in range(20):
                b.run(sv, dY, X, nbr, Wt, s2)
            s2.synchronize()
        except Exception as e:  # pragma: no cover - reported below
            errors.append(e)

    ts = [threading.Thread(target=capture), threading.Thread(target=eager)]
    for t in ts:
        t.start()
    for t in ts:
        t.join()
    assert not errors, errors
    torch.cuda.synchronize()
    assert b.equal(ref), "eager calls on the second stream changed"
    g.replay()
    torch.cuda.synchronize()
    assert a.equal(ref), "captured calls differ from a plain call"

    # a capture on a stream that never had a side stream: the launches run in order on it
    g3 = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g3, stream=s3, capture_error_mode="thread_local"):
        c.run(sv, dY, X, nbr, Wt, s3)
    g3.replay()
    torch.cuda.synchronize()
    assert c.equal(ref), "capture without a side stream differs from a plain call"
    assert sv.svconv_read_error_word() == 0
    del g, g3
