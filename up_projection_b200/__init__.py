"""B200 (sm_100a) fused SwiGLU gate/up projection.

The Python layer is argument marshalling only: every step of the forward and
backward runs in the CUDA kernels of ``libswiglu_b200.so`` behind the C ABI
declared in ``include/swiglu.h``.  Importing this package does not load the
library; the first call does, and raises if it is missing or cannot run.
"""
from ._capi import (  # noqa: F401
    SWIGLU_ACT_GELU_TANH, SWIGLU_ACT_SILU, SWIGLU_BF16, SWIGLU_FP32, SwigluError, dswiglu_bwd, lib, status_string,
    swiglu_bwd_dw, swiglu_bwd_dx, swiglu_bwd_gemms, swiglu_fwd, swiglu_fwd_fp8, swiglu_last_route, swiglu_read_floor, swiglu_route_for,
    swiglu_sync_status,
)
