"""SALR sparse + low-rank linear layer for NVIDIA B200 (sm_100a).

``Y = X (M (.) W)^T + (X A_cat) B_cat`` with W magnitude-pruned per row and stored as a
bitmap plus compact values; one hand-written CUDA kernel per call.  The Python layer is
a ctypes binding of the C ABI in ``include/salr.h``; importing it does not load the
library, the first call does (and fails loudly if it has not been built).
"""
from .binding import (SIGNATURES, SalrError, SalrPlan, Weight, encode, linear, linear_host,
                      load, load_library, plan, residual_adapter, status_string)

__all__ = ["SIGNATURES", "SalrError", "SalrPlan", "Weight", "encode", "linear", "linear_host",
           "load", "load_library", "plan", "residual_adapter", "status_string"]
