"""Tree-indexed sparse attention (Zyphra Hierarchical Attention's hot path) for
NVIDIA B200: C-ABI CUDA library (libzha.so) plus a thin ctypes binding.

    from hierarchical_tree_indexed_b200 import zha        # the binding
    from hierarchical_tree_indexed_b200 import workloads  # seeded inputs

Importing the package loads nothing; the first library call loads libzha.so
and raises if it is missing.
"""
