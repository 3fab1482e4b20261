"""Dense-reconstruction baseline: the pipeline SparseConv2D replaces (a baseline, not the product).

The SV-TAD page (papernotes.org, "SV-TAD: Native Sparse Convolutions for Efficient Temporal
Action Detection", Background & Motivation) describes how convolutions over pruned tokens
are run without a native sparse operator: scatter the kept tokens back onto an empty dense
grid, run a standard zero-padded convolution over the whole grid, and gather the kept
positions again.  Key Findings puts the break-even point of the native operator against
dense convolution at a 55% keep rate.  This module is that dense pipeline, built from
PyTorch ops (index_copy / cuDNN conv2d in channels-last / index_select), so that the
crossover can be measured on the same GPU.  It is only ever timed beside the library's
kernels; nothing in the library calls it.
"""
from __future__ import annotations

import torch
import torch.nn.functional as F


def linear_cells(coords: torch.Tensor, H: int, W: int) -> torch.Tensor:
    """Row of each kept token in the dense [T * H * W] grid (int64)."""
    c = coords.long()
    return (c[:, 0] * H + c[:, 1]) * W + c[:, 2]


def torch_weight(Wt: torch.Tensor) -> torch.Tensor:
    """W [C_out][9][C_in] (taps row-major over (dy, dx)) -> conv2d weight [C_out][C_in][3][3]."""
    Cout, _, Cin = Wt.shape
    return Wt.view(Cout, 3, 3, Cin).permute(0, 3, 1, 2).contiguous(memory_format=torch.channels_last)


class DenseRecon:
    """Scatter -> dense 3x3 conv2d (zero padding) -> gather, for one token layout."""

    def __init__(self, coords: torch.Tensor, T: int, H: int, W: int):
        self.T, self.H, self.W = T, H, W
        self.cells = linear_cells(coords, H, W)

    def scatter(self, X: torch.Tensor) -> torch.Tensor:
        """Kept rows onto a zero grid, as an NCHW view in channels-last memory."""
        C = X.shape[1]
        G = torch.zeros((self.T * self.H * self.W, C), dtype=X.dtype, device=X.device)
        G.index_copy_(0, self.cells, X)
        return G.view(self.T, self.H, self.W, C).permute(0, 3, 1, 2)

    def gather(self, Yd: torch.Tensor) -> torch.Tensor:
        """Kept positions of a dense NCHW (channels-last) output, back to packed rows."""
        Cout = Yd.shape[1]
        flat = Yd.permute(0, 2, 3, 1).reshape(self.T * self.H * self.W, Cout)
        return flat.index_select(0, self.cells)

    def fwd(self, X: torch.Tensor, w_torch: torch.Tensor, bias=None) -> torch.Tensor:
        b = bias.to(X.dtype) if bias is not None else None
        return self.gather(F.conv2d(self.scatter(X), w_torch, b, padding=1))

    def fwd_bwd(self, X: torch.Tensor, w_torch: torch.Tensor, dY: torch.Tensor, bias=None):
        """Forward, then the gradients w.r.t. X, the weight and the bias by autograd through
        the same dense pipeline (gather -> scatter of dY, cuDNN data / weight gradients)."""
        Xr = X.detach().requires_grad_(True)
        wr = w_torch.detach().requires_grad_(True)
        br = (bias.detach().to(X.dtype).requires_grad_(True) if bias is not None else None)
        Y = self.gather(F.conv2d(self.scatter(Xr), wr, br, padding=1))
        gX, gW, *gb = torch.autograd.grad(Y, [Xr, wr] + ([br] if br is not None else []), dY)
        return Y.detach(), gX, gW, (gb[0] if gb else None)
