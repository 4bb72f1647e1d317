"""Lookahead Sparse Attention (LSA) decode hot path for NVIDIA B200 (sm_100a).

The kernels live in liblsa.so (C ABI: include/lsa.h); ``lsa`` is its thin
ctypes binding.  Build with ``python -m lookahead_sparse_kv_index_b200.build``.
"""
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "liblsa.so")
