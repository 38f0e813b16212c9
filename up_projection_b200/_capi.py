"""ctypes binding of libswiglu_b200.so (the C ABI of include/swiglu.h).

Argument marshalling only: torch tensors become device pointers and the
current CUDA stream becomes a cudaStream_t; the library does all the work.
The library is loaded on first use; if it is missing or cannot be loaded the
call raises -- there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libswiglu_b200.so")

# enum swiglu_dtype
SWIGLU_BF16 = 0
SWIGLU_FP32 = 1
# enum swiglu_status
SWIGLU_OK = 0
SWIGLU_ERR_NULL_POINTER = 1
SWIGLU_ERR_BAD_DIM = 2
SWIGLU_ERR_MISALIGNED_DIM = 3
SWIGLU_ERR_MISALIGNED_PTR = 4
SWIGLU_ERR_BAD_DTYPE = 5
SWIGLU_ERR_UNSUPPORTED_DEVICE = 6
SWIGLU_ERR_CUDA = 7
SWIGLU_ERR_TIMEOUT = 8
SWIGLU_ERR_OVERLAP = 9
SWIGLU_ERR_NO_DEVICE = 10
SWIGLU_ERR_BAD_FLAGS = 11
SWIGLU_ERR_BAD_EPILOGUE = 12
# enum swiglu_activation
SWIGLU_ACT_SILU = 0
SWIGLU_ACT_GELU_TANH = 1
# enum swiglu_flags
SWIGLU_FLAG_WEIGHTS_STABLE = 1
# enum swiglu_route
ROUTE_NONE = 0
ROUTE_ZERO_K = 1
ROUTE_DECODE_BF16 = 2
ROUTE_GEMM_BF16 = 3
ROUTE_GEMM_TF32X3 = 4
ROUTE_BWD_GEMM_BF16 = 5
ROUTE_BWD_GEMM_TF32X3 = 6
ROUTE_STREAM_TC_BF16 = 7

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


class Epilogue(ctypes.Structure):
    """struct swiglu_epilogue."""
    _fields_ = [("activation", ctypes.c_int), ("gate_multiplier", ctypes.c_float),
                ("G", ctypes.c_void_p), ("U", ctypes.c_void_p)]


# name -> (restype, argtypes), mirroring include/swiglu.h
SIGNATURES = {
    "swiglu_fwd": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _I, _P]),
    "swiglu_fwd_ex": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _I, ctypes.c_uint, _P]),
    "swiglu_fwd_epilogue": (_I, [_P, _P, _P, _P, _I64, _I64, _I64, _I, ctypes.POINTER(Epilogue),
                                 ctypes.c_uint, _P]),
    "dswiglu_bwd_epilogue": (_I, [_P, _P, _P, _P, _P, _I64, _I, _I, ctypes.c_float, _P]),
    "dswiglu_bwd": (_I, [_P, _P, _P, _P, _P, _I64, _P]),
    "dswiglu_bwd_dtype": (_I, [_P, _P, _P, _P, _P, _I64, _I, _P]),
    "swiglu_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, ctypes.POINTER(Epilogue), _P]),
    "swiglu_bwd_dx": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P]),
    "swiglu_bwd_dx_noalloc": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P]),
    "swiglu_bwd_dw": (_I, [_P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P]),
    "swiglu_bwd_gemms": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I, _P]),
    "swiglu_route_for": (_I, [_I64, _I64, _I64, _I]),
    "swiglu_last_route": (_I, []),
    "swiglu_status_string": (ctypes.c_char_p, [_I]),
    "swiglu_sync_status": (_I, [_P]),
    "swiglu_read_floor": (_I, [_P, _P, _I64, _P, _P]),
    "swiglu_selftest_wait_timeout": (_I, [_P]),
    "swiglu_read_floor_sink_words": (_I64, []),
}

_lock = threading.Lock()
_lib = None


class SwigluError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """The loaded library (raises if it is not built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m up_projection_b200.build` (nvcc, sm_100a)")
            handle = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                f = getattr(handle, name)
                f.restype = res
                f.argtypes = args
            _lib = handle
    return _lib


def status_string(status: int) -> str:
    return lib().swiglu_status_string(int(status)).decode()


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _check(fn: str, st: int):
    if st != SWIGLU_OK:
        raise SwigluError(fn, st)


_DT = {torch.bfloat16: SWIGLU_BF16, torch.float32: SWIGLU_FP32}


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype not in _DT:
        raise TypeError(f"unsupported dtype {t.dtype}; use bfloat16 or float32")
    return _DT[t.dtype]


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def swiglu_fwd(X: torch.Tensor, Wg: torch.Tensor, Wu: torch.Tensor,
               H: torch.Tensor | None = None, stream=None,
               weights_stable: bool = False, activation: int = SWIGLU_ACT_SILU,
               gate_multiplier: float = 1.0, return_gu: bool = False):
    """H = silu(X Wg^T) * (X Wu^T) through the C ABI.  X [..., K] (leading
    dims are flattened to M rows, as the TensorRT-LLM fused up-projection
    does), Wg/Wu [N, K]; bf16 or fp32, all contiguous on one GPU.

    weights_stable=True promises that no earlier work on the stream writes
    Wg or Wu (SWIGLU_FLAG_WEIGHTS_STABLE): the weight-streaming kernels (bf16
    decode at M <= 8, the tcgen05 stream at 9 <= M <= 128) may then start
    streaming them while the preceding kernel finishes.

    activation / gate_multiplier select the epilogue variant
    H = act(gate_multiplier * G) * U (SWIGLU_ACT_SILU or
    SWIGLU_ACT_GELU_TANH).  return_gu=True also stores G = X Wg^T and
    U = X Wu^T (training forward) and returns (H, G, U)."""
    # (the checks are ordered for the per-call cost of the decode path: one
    # pass of cheap attribute reads, the detailed messages only on failure)
    if not (X.is_cuda and Wg.is_cuda and Wu.is_cuda and X.is_contiguous()
            and Wg.is_contiguous() and Wu.is_contiguous()):
        for t, n in ((X, "X"), (Wg, "Wg"), (Wu, "Wu")):
            _dev(t, n)
    dt = X.dtype
    if Wg.dtype != dt or Wu.dtype != dt:
        raise TypeError("X, Wg and Wu must share a dtype")
    code = _DT.get(dt)
    if code is None:
        _dtype_code(X)
    xs = X.shape
    K = xs[-1]
    ws = Wg.shape
    N = ws[0]
    if len(ws) != 2 or ws[1] != K or Wu.shape != ws:
        raise ValueError(f"weights must be [N, K] = [{N}, {K}]")
    M = X.numel() // K if K else math.prod(xs[:-1])
    if H is None:
        H = torch.empty((*xs[:-1], N), dtype=dt, device=X.device)
    elif not (H.is_cuda and H.is_contiguous()):
        _dev(H, "H")
    elif H.dtype != dt or H.numel() != M * N:
        raise ValueError("H has the wrong dtype or size")
    flags = SWIGLU_FLAG_WEIGHTS_STABLE if weights_stable else 0
    G = U = None
    if return_gu:
        G = torch.empty_like(H)
        U = torch.empty_like(H)
    if activation == SWIGLU_ACT_SILU and gate_multiplier == 1.0 and not return_gu:
        st = lib().swiglu_fwd_ex(X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), H.data_ptr(),
                                 M, K, N, code, flags, _stream(stream))
    else:
        epi = Epilogue(int(activation), float(gate_multiplier),
                       G.data_ptr() if G is not None else None,
                       U.data_ptr() if U is not None else None)
        st = lib().swiglu_fwd_epilogue(X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), H.data_ptr(),
                                       M, K, N, code, ctypes.byref(epi), flags,
                                       _stream(stream))
    _check("swiglu_fwd", st)
    return (H, G, U) if return_gu else H


def dswiglu_bwd(dH: torch.Tensor, G: torch.Tensor, U: torch.Tensor,
                dG: torch.Tensor | None = None, dU: torch.Tensor | None = None,
                stream=None, activation: int = SWIGLU_ACT_SILU, gate_multiplier: float = 1.0):
    """(dG, dU) of h = act(gate_multiplier g) * u through the C ABI (bf16 or
    fp32); the defaults are the plain dSwiGLU."""
    for t, n in ((dH, "dH"), (G, "G"), (U, "U")):
        _dev(t, n)
    if not (dH.dtype == G.dtype == U.dtype) or dH.shape != G.shape or G.shape != U.shape:
        raise ValueError("dH, G, U must share dtype and shape")
    dG = torch.empty_like(G) if dG is None else dG
    dU = torch.empty_like(U) if dU is None else dU
    _dev(dG, "dG")
    _dev(dU, "dU")
    st = lib().dswiglu_bwd_epilogue(dH.data_ptr(), G.data_ptr(), U.data_ptr(), dG.data_ptr(),
                                    dU.data_ptr(), G.numel(), _dtype_code(G), int(activation),
                                    float(gate_multiplier), _stream(stream))
    _check("dswiglu_bwd", st)
    return dG, dU


def swiglu_fwd_fp8(X: torch.Tensor, Wg: torch.Tensor, Wu: torch.Tensor, stream=None,
                   activation: int = SWIGLU_ACT_SILU, gate_multiplier: float = 1.0):
    """Quantised forward through the C ABI: returns (Hq, Hs) with Hq the
    e4m3 codes [..., N] (torch.uint8) and Hs the UE8M0 scale codes
    [..., ceil(N/32)] (torch.uint8) of H = act(gate_multiplier G) U; the
    value of element n is e4m3(Hq) * 2^(Hs[n // 32] - 127).  bf16 inputs."""
    for t, n in ((X, "X"), (Wg, "Wg"), (Wu, "Wu")):
        _dev(t, n)
    if not (X.dtype == Wg.dtype == Wu.dtype == torch.bfloat16):
        raise TypeError("swiglu_fwd_fp8 takes bfloat16 X, Wg, Wu")
    K = X.shape[-1]
    N = Wg.shape[0]
    if Wg.shape != (N, K) or Wu.shape != (N, K):
        raise ValueError(f"weights must be [N, K] = [{N}, {K}]")
    lead = X.shape[:-1]
    M = 1
    for d in lead:
        M *= d
    Hq = torch.empty((*lead, N), dtype=torch.uint8, device=X.device)
    Hs = torch.empty((*lead, (N + 31) // 32), dtype=torch.uint8, device=X.device)
    epi = Epilogue(int(activation), float(gate_multiplier), None, None)
    st = lib().swiglu_fwd_fp8(X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), Hq.data_ptr(),
                              Hs.data_ptr(), M, K, N, ctypes.byref(epi), _stream(stream))
    _check("swiglu_fwd_fp8", st)
    return Hq, Hs


def _bwd_shapes(dG, dU, name_w, W):
    for t, n in ((dG, "dG"), (dU, "dU"), (W, name_w)):
        _dev(t, n)
    if not (dG.dtype == dU.dtype == W.dtype) or dG.dtype not in _DT:
        raise TypeError("the backward GEMMs take bfloat16 or float32 tensors of one dtype")
    if dG.shape != dU.shape:
        raise ValueError("dG and dU must have the same shape")
    N = dG.shape[-1]
    M = 1
    for d in dG.shape[:-1]:
        M *= d
    return M, N


def swiglu_bwd_dx(dG: torch.Tensor, dU: torch.Tensor, Wg: torch.Tensor, Wu: torch.Tensor,
                  dX: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """dX = dG Wg + dU Wu through the C ABI (bf16, or fp32 by 3xTF32).  dG, dU [..., N] (leading
    dims flattened to M rows), Wg, Wu [N, K]; dX has dG's leading dims."""
    M, N = _bwd_shapes(dG, dU, "Wg", Wg)
    _dev(Wu, "Wu")
    K = Wg.shape[-1]
    if Wg.shape != (N, K) or Wu.shape != (N, K) or Wu.dtype != Wg.dtype:
        raise ValueError(f"weights must be [N, K] = [{N}, {K}] of dG's dtype")
    if dX is None:
        dX = torch.empty((*dG.shape[:-1], K), dtype=dG.dtype, device=dG.device)
    else:
        _dev(dX, "dX")
        if dX.dtype != dG.dtype or dX.numel() != M * K:
            raise ValueError("dX has the wrong dtype or size")
    st = lib().swiglu_bwd_dx(dG.data_ptr(), dU.data_ptr(), Wg.data_ptr(), Wu.data_ptr(),
                             dX.data_ptr(), M, K, N, _dtype_code(dG), _stream(stream))
    _check("swiglu_bwd_dx", st)
    return dX


def swiglu_bwd_dw(dG: torch.Tensor, dU: torch.Tensor, X: torch.Tensor,
                  dWg: torch.Tensor | None = None, dWu: torch.Tensor | None = None,
                  stream=None):
    """(dWg, dWu) = (dG^T X, dU^T X) through the C ABI (bf16, or fp32 by 3xTF32).  dG, dU
    [..., N] and X [..., K] with the same leading dims (M rows)."""
    M, N = _bwd_shapes(dG, dU, "X", X)
    K = X.shape[-1]
    if X.numel() != M * K:
        raise ValueError("X must have dG's leading dims")
    dWg = torch.empty((N, K), dtype=X.dtype, device=X.device) if dWg is None else dWg
    dWu = torch.empty((N, K), dtype=X.dtype, device=X.device) if dWu is None else dWu
    for t, n in ((dWg, "dWg"), (dWu, "dWu")):
        _dev(t, n)
        if t.dtype != X.dtype or t.numel() != N * K:
            raise ValueError(f"{n} has the wrong dtype or size")
    st = lib().swiglu_bwd_dw(dG.data_ptr(), dU.data_ptr(), X.data_ptr(), dWg.data_ptr(),
                             dWu.data_ptr(), M, K, N, _dtype_code(dG), _stream(stream))
    _check("swiglu_bwd_dw", st)
    return dWg, dWu


def swiglu_bwd_gemms(dG: torch.Tensor, dU: torch.Tensor, Wg: torch.Tensor, Wu: torch.Tensor,
                     X: torch.Tensor, stream=None):
    """(dX, dWg, dWu) of the projection in one call (bf16 or fp32; for fp32
    one balanced launch runs all three GEMMs)."""
    M, N = _bwd_shapes(dG, dU, "Wg", Wg)
    for t, n in ((Wu, "Wu"), (X, "X")):
        _dev(t, n)
    K = Wg.shape[-1]
    if Wg.shape != (N, K) or Wu.shape != (N, K) or X.shape[-1] != K or X.numel() != M * K:
        raise ValueError("shapes: dG, dU [.., N], Wg, Wu [N, K], X [.., K] with dG's leading dims")
    if not (Wu.dtype == X.dtype == dG.dtype):
        raise TypeError("all tensors must share one dtype")
    dX = torch.empty((*dG.shape[:-1], K), dtype=dG.dtype, device=dG.device)
    dWg = torch.empty((N, K), dtype=dG.dtype, device=dG.device)
    dWu = torch.empty((N, K), dtype=dG.dtype, device=dG.device)
    st = lib().swiglu_bwd_gemms(dG.data_ptr(), dU.data_ptr(), Wg.data_ptr(), Wu.data_ptr(),
                                X.data_ptr(), dX.data_ptr(), dWg.data_ptr(), dWu.data_ptr(),
                                M, K, N, _dtype_code(dG), _stream(stream))
    _check("swiglu_bwd_gemms", st)
    return dX, dWg, dWu


def swiglu_route_for(M: int, K: int, N: int, dtype: int) -> int:
    return lib().swiglu_route_for(M, K, N, dtype)


def swiglu_last_route() -> int:
    return lib().swiglu_last_route()


def swiglu_sync_status(stream=None) -> int:
    return lib().swiglu_sync_status(_stream(stream))


def swiglu_read_floor(A: torch.Tensor, B: torch.Tensor, sink: torch.Tensor,
                      stream=None) -> None:
    """Bench-only: stream-read A and B (same byte size) once."""
    _dev(A, "A")
    _dev(B, "B")
    nbytes = A.numel() * A.element_size()
    if B.numel() * B.element_size() != nbytes:
        raise ValueError("A and B must have the same size in bytes")
    st = lib().swiglu_read_floor(A.data_ptr(), B.data_ptr(), nbytes, sink.data_ptr(),
                                 _stream(stream))
    _check("swiglu_read_floor", st)
