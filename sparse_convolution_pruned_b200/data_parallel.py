"""Data-parallel plumbing for the sparse convolution: frame shards and the gradient all-reduce.

Frames are independent (the neighbourhood is spatial only, within one frame), so a batch
of packed frames splits into contiguous frame ranges, one per rank, with no exchange for
the forward pass or the data gradient.  The weight and bias gradients are sums over
tokens, so the data-parallel gradient is the sum of the ranks' gradients: one all-reduce
of 9 * C_in * C_out + C_out fp32 values.  Host logic only; the kernels run through the
C ABI on each rank's shard.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class FrameShard:
    """Frames f0 .. f1 - 1 of the batch, i.e. packed tokens r0 .. r1 - 1."""
    f0: int
    f1: int
    r0: int
    r1: int
    coords: np.ndarray     # [r1 - r0, 3] int32, frame numbers rebased to 0 .. f1 - f0 - 1
    frame_off: np.ndarray  # [f1 - f0 + 1] int32, rebased to start at 0

    @property
    def T(self) -> int:
        return self.f1 - self.f0

    @property
    def n(self) -> int:
        return self.r1 - self.r0


def shard_frames(coords: np.ndarray, frame_off: np.ndarray, rank: int, world: int) -> FrameShard:
    """Contiguous frame range of `rank` out of `world` (frames split as evenly as possible)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a world of {world}")
    frame_off = np.asarray(frame_off, dtype=np.int64)
    T = frame_off.shape[0] - 1
    f0, f1 = T * rank // world, T * (rank + 1) // world
    r0, r1 = int(frame_off[f0]), int(frame_off[f1])
    c = np.array(np.asarray(coords)[r0:r1], dtype=np.int32, copy=True).reshape(-1, 3)
    c[:, 0] -= f0
    off = (frame_off[f0:f1 + 1] - r0).astype(np.int32)
    return FrameShard(f0, f1, r0, r1, c, off)


def allreduce_grads(grads, group=None):
    """Sum a flat fp32 gradient buffer (dW followed by db) over the ranks, in place."""
    import torch.distributed as dist

    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=group)
    return grads
