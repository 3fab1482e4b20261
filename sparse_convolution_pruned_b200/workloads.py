"""Seeded synthetic inputs for SparseConv2D on frame-wise pruned ViT tokens.

This module only draws random numbers and lays them out. It holds none of the
operator's arithmetic (no neighbour lookup, no convolution, no adapter math), so
both the CPU oracle side and the CUDA side of the tests consume exactly the same
bytes from here.

Token layout (shared by every consumer):
  * tokens are packed frame by frame; within a frame they are sorted by raster
    index y*W + x unless a caller shuffles them on purpose;
  * ``coords[k] = (t, y, x)`` as int32, ``frame_off[T+1]`` is CSR-style (frame t
    owns packed rows ``frame_off[t] .. frame_off[t+1]-1``);
  * features are row-major ``[n_kept][C]``; conv weights are ``W[C_out][9][C_in]``
    with tap ``j = (dy+1)*3 + (dx+1)``.

Keep patterns follow the workloads described for SV-TAD (papernotes.org, "SV-TAD:
Native Sparse Convolutions for Efficient Temporal Action Detection", Key Designs 1-2
and "Key Findings"): a ViT-L/16 style 16x16 patch grid per token-frame, with a fixed
number of tokens kept per frame.  Real pruning masks come from attention maps of a
trained backbone, which are not available; a blob-shaped saliency map with top-k
selection stands in for them (the kept sets are spatially clustered, like
attention-selected foreground, with ragged borders).

Notation ``N(0, s)`` below is mean 0 and variance s.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 samples to the nearest bfloat16 value (ties to even).

    Returns float32 values that are exactly representable in bf16, so converting
    them to bf16 later (``torch.bfloat16``) is exact.  Inputs are finite.
    """
    x = np.array(x, dtype=np.float32, copy=True, order="C")
    u = x.view(np.uint32)
    # finite inputs: u + 0x8000 stays below 2^32 (the largest finite pattern is 0xFF7FFFFF)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    u += np.uint32(0x7FFF)
    u += lsb
    u &= np.uint32(0xFFFF0000)
    return x


def round_to_e4m3(x: np.ndarray) -> np.ndarray:
    """Float32 samples rounded to the nearest value of the 8-bit float e4m3 (4 exponent, 3
    mantissa bits, largest finite 448), using torch's float8_e4m3fn conversion.  Returns
    float32 values exactly representable in e4m3.  Inputs lie well inside +-448."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).to(torch.float32).numpy()


def _normal(rng: np.random.Generator, shape, var: float, bf16: bool) -> np.ndarray:
    a = rng.standard_normal(size=shape, dtype=np.float32)
    if var != 1.0:
        a *= np.float32(np.sqrt(var))
    return round_to_bf16(a) if bf16 else a


def keep_uniform(rng: np.random.Generator, T: int, H: int, W: int, k: int) -> list:
    """Per frame, ``k`` raster indices drawn uniformly without replacement, sorted."""
    return [np.sort(rng.choice(H * W, size=k, replace=False)).astype(np.int64) for _ in range(T)]


def blob_saliency(rng: np.random.Generator, T: int, H: int, W: int) -> np.ndarray:
    """Per-frame saliency: sum of 3 Gaussian blobs (sigma ~ U(1.5, 4)) plus N(0, 0.1) noise.

    Blob centres are uniform on [0,H) x [0,W).  Shape [T, H, W], float64.
    """
    mu_y = rng.uniform(0.0, H, size=(T, 3))
    mu_x = rng.uniform(0.0, W, size=(T, 3))
    sig = rng.uniform(1.5, 4.0, size=(T, 3))
    eps = rng.standard_normal(size=(T, H, W)) * np.sqrt(0.1)
    yy = np.arange(H, dtype=np.float64)[None, :, None, None]
    xx = np.arange(W, dtype=np.float64)[None, None, :, None]
    d2 = (yy - mu_y[:, None, None, :]) ** 2 + (xx - mu_x[:, None, None, :]) ** 2
    s = np.exp(-d2 / (2.0 * sig[:, None, None, :] ** 2)).sum(axis=3)
    return s + eps


def keep_topk(sal: np.ndarray, ks) -> list:
    """Keep the top-k_t cells of each frame's saliency (ties to the lower raster index)."""
    T, H, W = sal.shape
    out = []
    for t in range(T):
        flat = sal[t].reshape(-1)
        order = np.argsort(-flat, kind="stable")
        out.append(np.sort(order[: int(ks[t])]).astype(np.int64))
    return out


def pack_tokens(keep: list, H: int, W: int):
    """Raster indices per frame -> (coords [n,3] int32, frame_off [T+1] int32)."""
    T = len(keep)
    off = np.zeros(T + 1, dtype=np.int64)
    for t in range(T):
        off[t + 1] = off[t] + len(keep[t])
    n = int(off[-1])
    coords = np.zeros((n, 3), dtype=np.int32)
    for t in range(T):
        r = keep[t]
        coords[off[t]:off[t + 1], 0] = t
        coords[off[t]:off[t + 1], 1] = r // W
        coords[off[t]:off[t + 1], 2] = r % W
    return coords, off.astype(np.int32)


@dataclass
class ConvWorkload:
    """One SparseConv2D problem: tokens plus conv operands (float32 arrays).

    For ``dtype == "bf16"`` every float array holds values exactly representable
    in bf16 (the bias stays fp32).
    """
    name: str
    T: int
    H: int
    W: int
    coords: np.ndarray
    frame_off: np.ndarray
    Cin: int
    Cout: int
    dtype: str
    X: np.ndarray
    Wt: np.ndarray
    bias: Optional[np.ndarray]
    dY: np.ndarray
    seed: int = 0
    notes: dict = field(default_factory=dict)

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])


@dataclass
class AdapterWorkload:
    """Bottleneck adapter: Linear D->R, SparseConv2D 3x3 R->R, GELU, Linear R->D, residual."""
    name: str
    T: int
    H: int
    W: int
    coords: np.ndarray
    frame_off: np.ndarray
    D: int
    R: int
    X: np.ndarray       # [n, D] bf16 values
    Wd: np.ndarray      # [R, D]
    Wc: np.ndarray      # [R, 9, R]
    Wu: np.ndarray      # [D, R]
    seed: int = 0

    @property
    def n(self) -> int:
        return int(self.coords.shape[0])


def conv_workload(name: str, *, T: int, H: int, W: int, keep: list, Cin: int, Cout: int,
                  dtype: str, w_var: float, bias_var: Optional[float], rng: np.random.Generator,
                  seed: int) -> ConvWorkload:
    coords, off = pack_tokens(keep, H, W)
    n = coords.shape[0]
    bf = dtype == "bf16"
    X = _normal(rng, (n, Cin), 1.0, bf)
    Wt = _normal(rng, (Cout, 9, Cin), w_var, bf)
    bias = None
    if bias_var is not None:
        bias = _normal(rng, (Cout,), bias_var, False)
    dY = _normal(rng, (n, Cout), 1.0, bf)
    return ConvWorkload(name, T, H, W, coords, off, Cin, Cout, dtype, X, Wt, bias, dY, seed)


def tiny_f32(seed: int = 0) -> ConvWorkload:
    """T=4, 8x8 grid, exactly 32 kept per frame (uniform), C=16, fp32; b ~ N(0, 0.1)."""
    rng = np.random.default_rng(seed)
    keep = keep_uniform(rng, 4, 8, 8, 32)
    return conv_workload("tiny_f32_T4_8x8_k32_C16", T=4, H=8, W=8, keep=keep, Cin=16, Cout=16,
                         dtype="f32", w_var=1.0, bias_var=0.1, rng=rng, seed=seed)


def small_c_bf16(seed: int = 1, T: int = 384, C: int = 64, k: int = 77) -> ConvWorkload:
    """16x16 grid, blob saliency, top-77 per frame (~30%), C_in=C_out=64, bf16, no bias."""
    rng = np.random.default_rng(seed)
    sal = blob_saliency(rng, T, 16, 16)
    keep = keep_topk(sal, [k] * T)
    return conv_workload(f"small_c_bf16_T{T}_16x16_k{k}_C{C}", T=T, H=16, W=16, keep=keep,
                         Cin=C, Cout=C, dtype="bf16", w_var=1.0 / (9 * C), bias_var=None,
                         rng=rng, seed=seed)


def large_c_fwd_bf16(seed: int = 2, T: int = 384, C: int = 256) -> ConvWorkload:
    """16x16 grid, blob saliency, keep 50% per frame, C=256, bf16, fp32 bias ~ N(0, 0.1)."""
    rng = np.random.default_rng(seed)
    sal = blob_saliency(rng, T, 16, 16)
    keep = keep_topk(sal, [128] * T)
    return conv_workload(f"large_c_fwd_bf16_T{T}_16x16_keep50_C{C}", T=T, H=16, W=16, keep=keep,
                         Cin=C, Cout=C, dtype="bf16", w_var=1.0 / (9 * C), bias_var=0.1,
                         rng=rng, seed=seed)


def large_c_fwd_e4m3(seed: int = 2, T: int = 384, C: int = 256) -> ConvWorkload:
    """The large-channel forward workload with X and W rounded to e4m3 (8-bit inference)."""
    w = large_c_fwd_bf16(seed=seed, T=T, C=C)
    w.X = round_to_e4m3(w.X)
    w.Wt = round_to_e4m3(w.Wt)
    w.dtype = "e4m3"
    w.name = f"large_c_fwd_e4m3_T{T}_16x16_keep50_C{C}"
    return w


def large_c_bwd_bf16(seed: int = 3, T: int = 384, C: int = 256) -> ConvWorkload:
    """As the large-channel forward, but the keep ratio r_t ~ U(0.2, 0.8) varies per frame."""
    rng = np.random.default_rng(seed)
    r = rng.uniform(0.2, 0.8, size=T)
    ks = np.rint(r * 256).astype(np.int64)
    sal = blob_saliency(rng, T, 16, 16)
    keep = keep_topk(sal, ks)
    return conv_workload(f"large_c_bwd_bf16_T{T}_16x16_keepU(0.2,0.8)_C{C}", T=T, H=16, W=16,
                         keep=keep, Cin=C, Cout=C, dtype="bf16", w_var=1.0 / (9 * C),
                         bias_var=0.1, rng=rng, seed=seed)


def adapter_bf16(seed: int = 4, T: int = 3072, D: int = 1024, R: int = 256) -> AdapterWorkload:
    """Long-video bottleneck adapter: 16x16 grid, keep 36% (92 per frame), D=1024, R=256."""
    rng = np.random.default_rng(seed)
    k = int(round(0.36 * 256))
    sal = blob_saliency(rng, T, 16, 16)
    keep = keep_topk(sal, [k] * T)
    coords, off = pack_tokens(keep, 16, 16)
    n = coords.shape[0]
    X = _normal(rng, (n, D), 1.0, True)
    Wd = _normal(rng, (R, D), 1.0 / D, True)
    Wc = _normal(rng, (R, 9, R), 1.0 / (9 * R), True)
    Wu = _normal(rng, (D, R), 1.0 / R, True)
    return AdapterWorkload(f"adapter_bf16_T{T}_16x16_keep36_D{D}_R{R}", T, 16, 16, coords, off,
                           D, R, X, Wd, Wc, Wu, seed)


def custom_conv(*, seed: int, T: int, H: int, W: int, keep_frac, Cin: int, Cout: int, dtype: str,
                bias: bool = True, shuffle: bool = False, empty_frames=()) -> ConvWorkload:
    """Edge-case generator: uniform random keep with a per-frame fraction (float or list).

    ``empty_frames`` lists frames that keep nothing; ``shuffle`` permutes tokens
    inside each frame (frames stay contiguous).
    """
    rng = np.random.default_rng(seed)
    fr = keep_frac if isinstance(keep_frac, (list, tuple, np.ndarray)) else [keep_frac] * T
    keep = []
    for t in range(T):
        k = 0 if t in empty_frames else max(0, min(H * W, int(round(fr[t] * H * W))))
        sel = rng.choice(H * W, size=k, replace=False)
        sel = sel if shuffle else np.sort(sel)
        keep.append(sel.astype(np.int64))
    bf = dtype == "bf16"
    wv = 1.0 / (9 * Cin) if bf else 1.0
    return conv_workload(f"custom_T{T}_{H}x{W}_C{Cin}x{Cout}_{dtype}", T=T, H=H, W=W, keep=keep,
                         Cin=Cin, Cout=Cout, dtype=dtype, w_var=wv, bias_var=0.1 if bias else None,
                         rng=rng, seed=seed)


CONFIGS = {
    "tiny_f32": tiny_f32,
    "small_c_bf16": small_c_bf16,
    "large_c_fwd_bf16": large_c_fwd_bf16,
    "large_c_fwd_e4m3": large_c_fwd_e4m3,
    "large_c_bwd_bf16": large_c_bwd_bf16,
    "adapter_bf16": adapter_bf16,
}
