"""ZHA (Zyphra Hierarchical Attention) decode path for B200 (sm_100a).

The compute lives in libzha.so (C ABI, include/zha.h); ``zha`` is its thin
Python binding and ``inputs`` the seeded synthetic-input generator. Importing
the package does not load the CUDA library; ``from tree_indexed_sparse_02_b200
import zha`` does, and fails loudly if it is not built.
"""
