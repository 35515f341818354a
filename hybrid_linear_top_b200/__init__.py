"""LISA (Linear-Indexed Sparse Attention) for B200 / sm_100a.

The layer's kernels live in liblisa.so (C ABI in include/lisa.h); the
submodule ``lisa`` binds it with ctypes.  Importing ``hybrid_linear_top_b200.lisa``
loads the library and raises if it has not been built.
"""

__all__ = ["lisa"]
