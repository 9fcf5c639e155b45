"""B200-native LongCat Sparse Attention (LSA) layer hot path.

The CUDA kernels and the C-ABI live in ``csrc/`` and build into ``liblsa.so`` in this
directory; ``lsa`` is the thin ctypes binding with the same entry-point names; ``workloads``
holds the seeded synthetic input recipes.  Importing the package loads nothing native.
"""
__all__ = ["lsa", "workloads"]
