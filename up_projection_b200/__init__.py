"""B200 (sm_100a) fused SwiGLU gate/up projection.

The Python layer is argument marshalling only: every step of the forward and
backward runs in the CUDA kernels of ``libswiglu_b200.so`` behind the C ABI
declared in ``include/swiglu.h``.  Importing this package does not load the
library; the first call does, and raises if it is missing or cannot run.
"""
