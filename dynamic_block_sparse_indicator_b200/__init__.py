"""Prism dynamic block-sparse video self-attention for NVIDIA B200 (sm_100a).

The compute lives in libprism.so (CUDA kernels behind the C ABI declared in
include/prism.h); this package is the thin Python binding over it.  There is
no CPU fallback: calls fail loudly when the library is missing or no sm_100
device is present.
"""
from ._lib import (PRISM_BF16, PRISM_F32, Plan, PrismError, PrismParams, load, make_params,
                   plan, plan_import, status_string, workspace_bytes)

__all__ = ["PRISM_BF16", "PRISM_F32", "Plan", "PrismError", "PrismParams", "load", "make_params",
           "plan", "plan_import", "status_string", "workspace_bytes"]
