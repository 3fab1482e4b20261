"""B200-native SparseConv2D on frame-wise pruned ViT tokens (SV-TAD hot path).

``svconv`` is the Python binding of the C-ABI CUDA library (loaded on first
use; it raises if the library is missing or no CUDA device is present).
``workloads`` holds the seeded synthetic input generators.
"""
__all__ = ["svconv", "workloads"]
