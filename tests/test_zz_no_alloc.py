"""The allocation-free weight-gradient entry point (svconv_bwd_weight_noalloc).

It exists for callers that cannot allocate device memory when they call the
library (fixed-budget services, plugins without access to their host's
allocator, callbacks where cudaMalloc would synchronise): its split partials
live in a fixed device array inside the library instead of a caller workspace.

Called here through the C ABI with raw device pointers, twice in a row with
different inputs, and compared with the ordinary entry point (bit for bit where
both use the same token splits) or, where the fixed array forces fewer splits,
with the oracle within the tests' bf16 tolerance.  This file is collected
last so a failure here does not hide others.
"""
import ctypes

import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl

pytestmark = pytest.mark.gpu

BF16_TOL = 2e-2


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


@pytest.mark.parametrize("make,dtype,same_splits", [
    (lambda: wl.small_c_bf16(), torch.bfloat16, True),            # partials fit: the usual splits
    (lambda: wl.large_c_bwd_bf16(T=48), torch.bfloat16, False),   # C=256: fewer splits than usual
    (lambda: wl.tiny_f32(), torch.float32, True),
], ids=["small_c_bf16", "c256_fewer_splits", "tiny_f32"])
def test_noalloc_matches_workspace_entry_point_twice(sv, make, dtype, same_splits):
    """Two calls in a row with different dY.  Where the usual split count fits the fixed
    array, the two entry points run the same kernels with the same splits and must agree
    bit for bit (a wrong partial-row offset inside the array would show); with fewer
    splits the summation order differs, so that case is held to the oracle instead."""
    w = make()
    nbr, _ = sv.svconv_build_index(_dev(w.coords), _dev(w.frame_off), w.T, w.H, w.W)
    X = _dev(w.X, dtype)
    code = sv.BF16 if dtype == torch.bfloat16 else sv.F32
    rng = np.random.default_rng(99)
    if not same_splits:
        import oracle
        oracle.build()
        ref_nbr = nbr.cpu().numpy()
    for call in range(2):  # two calls in a row, different dY each time
        dY_np = w.dY if call == 0 else wl.round_to_bf16(rng.standard_normal(w.dY.shape).astype(np.float32))
        dY = _dev(dY_np, dtype)
        dW, db = _noalloc(sv, code, dY, X, nbr, w.Cin, w.Cout)
        torch.cuda.synchronize()
        assert torch.isfinite(dW).all() and torch.isfinite(db).all()
        if same_splits:
            ref_dW, ref_db = sv.svconv_bwd_weight(dY, X, nbr)
            torch.cuda.synchronize()
            assert torch.equal(dW, ref_dW) and torch.equal(db, ref_db)
        else:
            r_dW, r_db = oracle.bwd_weight(dY_np, w.X, ref_nbr)
            for got, ref in ((dW, r_dW), (db, r_db)):
                g = got.cpu().double().numpy()
                assert np.abs(g - ref).max() <= BF16_TOL * np.abs(ref).max()
    assert sv.svconv_read_error_word() == 0


def test_noalloc_second_call_takes_no_device_memory(sv):
    """After a first call has committed the fixed array, a further call leaves the
    device's free memory unchanged (it allocates nothing)."""
    w = wl.small_c_bf16()
    nbr, _ = sv.svconv_build_index(_dev(w.coords), _dev(w.frame_off), w.T, w.H, w.W)
    X = _dev(w.X, torch.bfloat16)
    dY = _dev(w.dY, torch.bfloat16)
    dW = torch.empty((w.Cout, 9, w.Cin), device="cuda")
    db = torch.empty((w.Cout,), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (sv.BF16, _p(dY), _p(X), _p(nbr), w.n, w.Cin, w.Cout, _p(dW), _p(db), stream)
    assert sv.lib().svconv_bwd_weight_noalloc(*args) == 0
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    assert sv.lib().svconv_bwd_weight_noalloc(*args) == 0
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0


def test_noalloc_empty_call_is_accepted(sv):
    """An empty call (n = 0) succeeds and zeroes the gradients."""
    dW = torch.full((64, 9, 64), float("nan"), device="cuda")
    db = torch.full((64,), float("nan"), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = sv.lib().svconv_bwd_weight_noalloc(sv.BF16, None, None, None, 0, 64, 64, _p(dW), _p(db), stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert (dW == 0).all() and (db == 0).all()


def test_noalloc_rejects_channels_beyond_the_scratch(sv):
    # one split of C_in = C_out = 1024 needs 16 x 640 = 10240 partial rows x 1024 floats = 40 MiB > 16 MiB
    X = torch.zeros((64, 1024), dtype=torch.bfloat16, device="cuda")
    nbr = torch.full((64, 9), -1, dtype=torch.int32, device="cuda")
    dW = torch.empty((1024, 9, 1024), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = sv.lib().svconv_bwd_weight_noalloc(sv.BF16, _p(X), _p(X), _p(nbr), 64, 1024, 1024, _p(dW), None, stream)
    assert rc == -2  # SVCONV_ERR_SIZE
