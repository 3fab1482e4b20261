"""The allocation-free weight-gradient entry point (svconv_bwd_weight_noalloc).

It exists for callers that cannot allocate device memory when they call the
library (fixed-budget services, plugins without access to their host's
allocator, callbacks where cudaMalloc would synchronise): its split partials
live in a fixed device array inside the library instead of a caller workspace.

Called here through the C ABI with raw device pointers, twice in a row with
different inputs, and compared with the ordinary entry point within the tests'
tolerance.  This file is collected last so a failure here does not hide others.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2
F32_TOL = 1e-5


@pytest.fixture(scope="module")
def sv():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from sparse_convolution_pruned_b200 import build, svconv
    build.build()
    L = svconv.lib()
    L.svconv_bwd_weight_noalloc.argtypes = [ctypes.c_int] + [ctypes.c_void_p] * 3 + [ctypes.c_int] * 3 + \
        [ctypes.c_void_p] * 3
    L.svconv_bwd_weight_noalloc.restype = ctypes.c_int
    return svconv


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(sv, dtype_code, dY, X, nbr, Cin, Cout):
    dW = torch.full((Cout, 9, Cin), float("nan"), device="cuda")
    db = torch.full((Cout,), float("nan"), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = sv.lib().svconv_bwd_weight_noalloc(dtype_code, _p(dY), _p(X), _p(nbr), dY.shape[0], Cin, Cout,
                                            _p(dW), _p(db), stream)
    assert rc == 0, sv.status_str(rc)
    return dW, db


def _dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.to(dtype) if dtype is not None else t).cuda()


@pytest.mark.parametrize("make,dtype", [
    (lambda: wl.small_c_bf16(), torch.bfloat16),               # partials fit: the usual splits
    (lambda: wl.large_c_bwd_bf16(T=48), torch.bfloat16),       # C=256: fewer splits than usual
    (lambda: wl.tiny_f32(), torch.float32),
], ids=["small_c_bf16", "c256_fewer_splits", "tiny_f32"])
def test_noalloc_matches_workspace_entry_point_twice(sv, make, dtype):
    w = make()
    nbr, _ = sv.svconv_build_index(_dev(w.coords), _dev(w.frame_off), w.T, w.H, w.W)
    X = _dev(w.X, dtype)
    code = sv.BF16 if dtype == torch.bfloat16 else sv.F32
    tol = BF16_TOL if dtype == torch.bfloat16 else F32_TOL
    rng = np.random.default_rng(99)
    for call in range(2):  # two calls in a row, different dY each time
        dY_np = w.dY if call == 0 else wl.round_to_bf16(rng.standard_normal(w.dY.shape).astype(np.float32))
        dY = _dev(dY_np, dtype)
        ref_dW, ref_db = sv.svconv_bwd_weight(dY, X, nbr)
        dW, db = _noalloc(sv, code, dY, X, nbr, w.Cin, w.Cout)
        torch.cuda.synchronize()
        for got, ref in ((dW, ref_dW), (db, ref_db)):
            g = got.cpu().double().numpy()
            r = ref.cpu().double().numpy()
            assert np.isfinite(g).all()
            if dtype == torch.bfloat16:
                assert np.abs(g - r).max() <= tol * np.abs(r).max()
            else:
                assert (np.abs(g - r) <= tol * (1 + np.abs(r))).all()
    assert sv.svconv_read_error_word() == 0


def test_noalloc_rejects_channels_beyond_the_scratch(sv):
    # one split of C_in = C_out = 1024 needs 16 x 640 = 10240 partial rows x 1024 floats = 40 MiB > 16 MiB
    X = torch.zeros((64, 1024), dtype=torch.bfloat16, device="cuda")
    nbr = torch.full((64, 9), -1, dtype=torch.int32, device="cuda")
    dW = torch.empty((1024, 9, 1024), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = sv.lib().svconv_bwd_weight_noalloc(sv.BF16, _p(X), _p(X), _p(nbr), 64, 1024, 1024, _p(dW), None, stream)
    assert rc == -2  # SVCONV_ERR_SIZE
