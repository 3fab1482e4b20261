"""The dense-reconstruction baseline (scatter -> conv2d -> gather) computes what the oracle
computes, so the keep-rate crossover compares two pipelines with the same result.

CPU: the baseline in float64 against the oracle (forward, data, weight and bias gradients).
GPU: the bf16 baseline (cuDNN) against the oracle within the bf16 bar.
"""
import numpy as np
import pytest
import torch

from sparse_convolution_pruned_b200 import workloads as wl
from sparse_convolution_pruned_b200.dense_recon import DenseRecon, torch_weight


def _case():
    return wl.custom_conv(seed=71, T=5, H=7, W=9, keep_frac=0.45, Cin=8, Cout=12, dtype="f32", shuffle=True,
                          empty_frames=(2,))


def test_dense_baseline_equals_oracle_fp64(orc):
    w = _case()
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).double()
    dense = DenseRecon(torch.from_numpy(w.coords), w.T, w.H, w.W)
    Y, gX, gW, gb = dense.fwd_bwd(d(w.X), torch_weight(d(w.Wt)), d(w.dY), d(w.bias))
    np.testing.assert_allclose(Y.numpy(), orc.fwd(w.X, ref_n, w.Wt, w.bias), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gX.numpy(), orc.bwd_data(w.dY, ref_n, w.Wt), rtol=1e-12, atol=1e-12)
    rdW, rdb = orc.bwd_weight(w.dY, w.X, ref_n)
    # conv2d weight gradient [C_out][C_in][3][3] -> W layout [C_out][9][C_in]
    got_dW = gW.permute(0, 2, 3, 1).reshape(w.Cout, 9, w.Cin).numpy()
    np.testing.assert_allclose(got_dW, rdW, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(gb.numpy(), rdb, rtol=1e-12, atol=1e-12)


@pytest.mark.gpu
def test_dense_baseline_bf16_on_gpu(orc):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    w = wl.small_c_bf16(T=24, C=64, k=140)
    ref_n, _, _ = orc.build_index(w.coords, w.frame_off, w.T, w.H, w.W, want_map=False)
    d = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    X, Wt, dY = d(w.X).bfloat16(), d(w.Wt).bfloat16(), d(w.dY).bfloat16()
    dense = DenseRecon(d(w.coords), w.T, w.H, w.W)
    Y, gX, gW, _ = dense.fwd_bwd(X, torch_weight(Wt), dY)
    torch.cuda.synchronize()
    for got, ref in ((Y.float().cpu().numpy(), orc.fwd(w.X, ref_n, w.Wt, None)),
                     (gX.float().cpu().numpy(), orc.bwd_data(w.dY, ref_n, w.Wt))):
        assert np.abs(got - ref).max() <= 2e-2 * np.abs(ref).max()
    rdW, _ = orc.bwd_weight(w.dY, w.X, ref_n)
    got_dW = gW.float().permute(0, 2, 3, 1).reshape(64, 9, 64).cpu().numpy()
    assert np.abs(got_dW - rdW).max() <= 2e-2 * np.abs(rdW).max()
