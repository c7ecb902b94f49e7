"""Qwen Sparse Attention (QSA) for B200 (sm_100a): CUDA kernels behind a C-ABI.

``block_sparse_long_09_b200.qsa`` is the Python binding of ``libqsa.so``;
``block_sparse_long_09_b200.inputs`` draws the seeded synthetic inputs.
Importing the package itself loads nothing.
"""
