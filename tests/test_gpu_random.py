"""Seeded random sweep of the whole path against the oracle (through the C ABI).

Each case draws a grid (1..21 x 1..21, tall, wide and one-row grids included), a number of
frames, per-frame keep fractions (empty and fully kept frames included), optional shuffling of
tokens inside frames, a dtype and channel widths, then checks the index build bit for bit and
the forward, data gradient and weight / bias gradients within the workload bars.  The draws are
fixed by the seed, so a failure names a reproducible case.
"""
import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_TOL = 2e-2


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_convolution_pruned_b200 import build, svconv
    build.build()
    return svconv


def draw_case(i):
    rng = np.random.default_rng(1000 + i)
    H, W = int(rng.integers(1, 22)), int(rng.integers(1, 22))
    T = int(rng.integers(1, 9))
    fr = rng.uniform(0.0, 1.0, size=T)
    fr[rng.random(T) < 0.15] = 0.0   # empty frames
    fr[rng.random(T) < 0.15] = 1.0   # fully kept frames
    if rng.random() < 0.5:
        dtype = "bf16"
        Cin = int(rng.choice([64, 128, 192, 256]))
        Cout = int(rng.choice([64, 128, 256, 320]))
    else:
        dtype = "f32"
        Cin = int(rng.integers(1, 9)) * 4
        Cout = int(rng.integers(1, 9)) * 4
    return dict(seed=2000 + i, T=T, H=H, W=W, keep_frac=list(fr), Cin=Cin, Cout=Cout, dtype=dtype,
                shuffle=bool(rng.random() < 0.5), bias=bool(rng.random() < 0.5))


@pytest.mark.parametrize("i", range(24))
def test_random_case(sv, orc, i):
    c = draw_case(i)
    w = wl.custom_conv(**c)
    d = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).to(dt) if dt else
                            torch.from_numpy(np.ascontiguousarray(a))).cuda()
    ref_n, ref_m, ref_st = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W)
    assert ref_st == 0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nbr, M = sv.svconv_build_index(d(w.coords), d(w.frame_off), w.T, w.H, w.W, want_map=True, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    np.testing.assert_array_equal(nbr.cpu().numpy(), ref_n)
    np.testing.assert_array_equal(M.cpu().numpy(), ref_m)
    if w.n == 0:
        return
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    X, Wt, dY = d(w.X, tdt), d(w.Wt, tdt), d(w.dY, tdt)
    b = d(w.bias) if w.bias is not None else None
    Y = sv.svconv_fwd(X, nbr, Wt, b)
    dX = sv.svconv_bwd_data(dY, nbr, Wt)
    dW, db = sv.svconv_bwd_weight(dY, X, nbr)
    dX2, dW2, db2 = sv.svconv_bwd(dY, X, nbr, Wt)
    torch.cuda.synchronize()
    assert torch.equal(dX, dX2)
    refs = [(Y, orc.fwd(w.X, ref_n, w.Wt, w.bias)), (dX, orc.bwd_data(w.dY, ref_n, w.Wt))]
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    refs += [(dW, rdW), (db, rdb), (dW2, rdW), (db2, rdb)]
    for got, ref in refs:
        g = got.float().cpu().numpy().astype(np.float64)
        if w.dtype == "bf16":
            assert np.abs(g - ref).max() <= BF16_TOL * np.abs(ref).max() + 1e-30, c
        else:
            assert (np.abs(g - ref) <= F32_TOL * (1 + np.abs(ref))).all(), c
    assert sv.svconv_read_error_word() == 0
