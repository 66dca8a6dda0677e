"""Importance-sampled block-sparse attention for B200 (sm_100a).

The compute path is the C-ABI library `libisa.so` (include/isa.h) built from
csrc/; `block_sparse_importance_b200.isa` is its thin ctypes binding.
`workloads` holds the seeded synthetic input generators.
Importing the package loads nothing; the CUDA library is loaded on first use
and its absence is an error, never a fallback.
"""
__all__ = ["isa", "workloads"]
