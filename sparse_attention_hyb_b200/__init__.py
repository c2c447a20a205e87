"""B200-native forward pass of one hybrid compressed attention layer (CSA / HCA,
flat and HISA indexers) — Python side of libhyb.

``abi`` is the ctypes binding of include/hyb.h (same entry-point names);
``layer`` composes the entry points with torch-allocated outputs and
workspaces.  All computation runs in libhyb's sm_100a kernels.
"""
from . import abi, layer  # noqa: F401
from .abi import (HYB_ATTN_DECODE, HYB_ATTN_PREFILL, HYB_ATTN_REAL_KV, HYB_DTYPE_BF16, HYB_DTYPE_F32,  # noqa: F401
                  HYB_INDEX_FLAT, HYB_INDEX_HISA, HybError)
