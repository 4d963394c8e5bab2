"""B200-native Lookahead Sparse Attention (LSA) decode step.

The hot path lives in ``liblsa.so`` (hand-written CUDA for sm_100a behind the C
ABI declared in ``include/lsa.h``).  ``learned_sparse_kv_b200.lsa`` is its
Python binding; ``learned_sparse_kv_b200.decode`` composes the calls into the
64-step lookahead window.
"""
from .build import LIB as LIB_PATH  # noqa: F401

__all__ = ["LIB_PATH"]
