"""C-ABI checks that need no GPU: the library loads, exports every function
include/swiglu.h declares, and validates arguments on the host before any
CUDA call (so the error codes are the same with or without a device)."""
import os
import re

import pytest

from up_projection_b200 import _capi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "swiglu.h")).read()
    return re.findall(r"SWIGLU_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


def test_header_declares_the_abi():
    names = declared_functions()
    assert {"swiglu_fwd", "dswiglu_bwd", "dswiglu_bwd_dtype"} <= set(names)


def test_library_exports_every_declared_symbol():
    lib = _capi.lib()
    for name in declared_functions():
        assert hasattr(lib, name), name
        assert name in _capi.SIGNATURES, f"binding lacks {name}"


def test_routes_are_a_pure_function_of_shape():
    r = _capi.swiglu_route_for
    assert r(8, 1536, 6912, 0) == _capi.ROUTE_DECODE_BF16
    assert r(1, 4096, 11008, 0) == _capi.ROUTE_DECODE_BF16
    for M in (9, 24, 64, 128):
        assert r(M, 4096, 11008, 0) == _capi.ROUTE_STREAM_TC_BF16
        assert r(M, 1536, 6912, 0) == _capi.ROUTE_STREAM_TC_BF16
    assert r(129, 4096, 11008, 0) == _capi.ROUTE_GEMM_BF16
    for M in (9, 12, 16, 17, 24, 25, 31, 32, 100, 128):
        for K, N in ((264, 72), (8, 8), (40, 1032), (2000, 264), (520, 6912)):
            # K not a multiple of 64
            assert r(M, K, N, 0) == _capi.ROUTE_GEMM_BF16, (M, K, N)
        for K, N in ((64, 8), (256, 512), (1536, 6912), (832, 1032), (4096, 264)):
            assert r(M, K, N, 0) == _capi.ROUTE_STREAM_TC_BF16, (M, K, N)
    assert r(8192, 4096, 14336, 0) == _capi.ROUTE_GEMM_BF16
    assert r(2048, 5120, 13824, 1) == _capi.ROUTE_GEMM_TF32X3
    assert r(8, 64, 64, 1) == _capi.ROUTE_GEMM_TF32X3
    assert r(4, 65536, 64, 0) == _capi.ROUTE_GEMM_BF16   # X stage too big for decode
    assert r(0, 64, 64, 0) == _capi.ROUTE_NONE
    assert r(4, 64, 0, 0) == _capi.ROUTE_NONE
    assert r(4, 0, 64, 0) == _capi.ROUTE_ZERO_K
    assert r(4, 60, 64, 0) == -1          # K not a multiple of 8 (bf16)
    assert r(4, 60, 64, 1) == _capi.ROUTE_GEMM_TF32X3   # multiple of 4 is fine for fp32
    assert r(4, 64, 66, 1) == -1
    assert r(-1, 64, 64, 0) == -1
    assert r(1 << 31, 64, 64, 0) == -1
    assert r(4, 64, 64, 2) == -1


@pytest.mark.parametrize("args,code", [
    ((None, None, None, None, 4, 64, 64, 0), _capi.SWIGLU_ERR_NULL_POINTER),
    ((16, 32, 48, 17, 4, 64, 64, 0), _capi.SWIGLU_ERR_MISALIGNED_PTR),
    ((16, 32, 48, 64, 4, 64, 64, 3), _capi.SWIGLU_ERR_BAD_DTYPE),
    ((16, 32, 48, 64, 4, 63, 64, 0), _capi.SWIGLU_ERR_MISALIGNED_DIM),
    ((16, 32, 48, 64, -4, 64, 64, 0), _capi.SWIGLU_ERR_BAD_DIM),
    # H [4,64] bf16 at 1 MiB overlaps X [4,64] placed inside it
    ((1 << 20, 1 << 24, 1 << 25, (1 << 20) - 16, 4, 64, 64, 0), _capi.SWIGLU_ERR_OVERLAP),
    ((None, None, None, None, 0, 64, 64, 0), _capi.SWIGLU_OK),
])
def test_fwd_host_validation(args, code):
    assert _capi.lib().swiglu_fwd(*args, None) == code


@pytest.mark.parametrize("args,code", [
    ((None, 16, 32, 48, 64, 10), _capi.SWIGLU_ERR_NULL_POINTER),
    ((16, 32, 48, 64, 80, -1), _capi.SWIGLU_ERR_BAD_DIM),
    ((16, 32, 48, 65, 80, 10), _capi.SWIGLU_ERR_MISALIGNED_PTR),
    ((1 << 20, 1 << 21, 1 << 22, 1 << 20, 1 << 23, 1000), _capi.SWIGLU_ERR_OVERLAP),  # dG == dH
    ((1 << 20, 1 << 21, 1 << 22, (1 << 21) + 16, 1 << 23, 1000), _capi.SWIGLU_ERR_OVERLAP),
    ((None, None, None, None, None, 0), _capi.SWIGLU_OK),
])
def test_bwd_host_validation(args, code):
    assert _capi.lib().dswiglu_bwd(*args, None) == code


def test_no_device_is_an_error_not_a_fallback():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _capi.lib().swiglu_fwd(1 << 20, 1 << 21, 1 << 22, 1 << 23, 4, 64, 64, 0, None)
    assert st == _capi.SWIGLU_ERR_NO_DEVICE


def test_unknown_flags_rejected():
    lib = _capi.lib()
    assert lib.swiglu_fwd_ex(16, 32, 48, 64, 4, 64, 64, 0, 2, None) == _capi.SWIGLU_ERR_BAD_FLAGS
    assert lib.swiglu_fwd_ex(None, None, None, None, 4, 64, 64, 0, 1, None) == \
        _capi.SWIGLU_ERR_NULL_POINTER


def test_epilogue_validation():
    import ctypes
    lib = _capi.lib()
    args = (1 << 20, 1 << 21, 1 << 22, 1 << 23, 4, 64, 64, 0)
    bad_act = _capi.Epilogue(7, 1.0, None, None)
    assert lib.swiglu_fwd_epilogue(*args, ctypes.byref(bad_act), 0, None) == \
        _capi.SWIGLU_ERR_BAD_EPILOGUE
    nan_mult = _capi.Epilogue(0, float("nan"), None, None)
    assert lib.swiglu_fwd_epilogue(*args, ctypes.byref(nan_mult), 0, None) == \
        _capi.SWIGLU_ERR_BAD_EPILOGUE
    only_g = _capi.Epilogue(0, 1.0, 1 << 24, None)
    assert lib.swiglu_fwd_epilogue(*args, ctypes.byref(only_g), 0, None) == \
        _capi.SWIGLU_ERR_BAD_EPILOGUE
    misaligned = _capi.Epilogue(0, 1.0, (1 << 24) + 8, 1 << 25)
    assert lib.swiglu_fwd_epilogue(*args, ctypes.byref(misaligned), 0, None) == \
        _capi.SWIGLU_ERR_MISALIGNED_PTR
    g_on_h = _capi.Epilogue(0, 1.0, 1 << 23, 1 << 25)   # G == H
    assert lib.swiglu_fwd_epilogue(*args, ctypes.byref(g_on_h), 0, None) == _capi.SWIGLU_ERR_OVERLAP
    g_on_x = _capi.Epilogue(0, 1.0, 1 << 20, 1 << 25)   # G == X
    assert lib.swiglu_fwd_epilogue(*args, ctypes.byref(g_on_x), 0, None) == _capi.SWIGLU_ERR_OVERLAP
    assert lib.dswiglu_bwd_epilogue(16, 32, 48, 64, 80, 10, 0, 5, 1.0, None) == \
        _capi.SWIGLU_ERR_BAD_EPILOGUE
    assert lib.dswiglu_bwd_epilogue(16, 32, 48, 64, 80, 10, 0, 1, float("inf"), None) == \
        _capi.SWIGLU_ERR_BAD_EPILOGUE


def test_status_strings():
    for code in range(13):
        assert _capi.status_string(code)
    assert _capi.status_string(999) == "unknown status"


# swiglu_bwd_dx(dG, dU, Wg, Wu, dX, M, K, N, dtype)
@pytest.mark.parametrize("args,code", [
    ((16, 32, 48, 64, None, 4, 64, 64, 0), _capi.SWIGLU_ERR_NULL_POINTER),
    ((None, 32, 48, 64, 80, 4, 64, 64, 0), _capi.SWIGLU_ERR_NULL_POINTER),
    ((16, 32, 48, 64, 88, 4, 64, 64, 0), _capi.SWIGLU_ERR_MISALIGNED_PTR),
    ((16, 32, 48, 64, 80, 4, 64, 64, 2), _capi.SWIGLU_ERR_BAD_DTYPE),
    ((16, 32, 48, 64, 80, 4, 60, 64, 0), _capi.SWIGLU_ERR_MISALIGNED_DIM),
    ((16, 32, 48, 64, 80, 4, 66, 64, 1), _capi.SWIGLU_ERR_MISALIGNED_DIM),   # fp32: K % 4
    ((16, 32, 48, 64, 80, 4, 64, 68, 0), _capi.SWIGLU_ERR_MISALIGNED_DIM),
    ((16, 32, 48, 64, 80, -1, 64, 64, 0), _capi.SWIGLU_ERR_BAD_DIM),
    ((16, 32, 48, 64, 80, 1 << 31, 64, 64, 0), _capi.SWIGLU_ERR_BAD_DIM),
    # dX [4,64] at 1 MiB overlaps Wg [64,64] placed 16 bytes before it
    ((1 << 22, 1 << 23, (1 << 20) - 16, 1 << 24, 1 << 20, 4, 64, 64, 0), _capi.SWIGLU_ERR_OVERLAP),
    ((1 << 20, 1 << 23, 1 << 22, 1 << 24, 1 << 20, 4, 64, 64, 0), _capi.SWIGLU_ERR_OVERLAP),
    ((None, None, None, None, None, 0, 64, 64, 0), _capi.SWIGLU_OK),   # M == 0
    ((None, None, None, None, None, 4, 0, 64, 0), _capi.SWIGLU_OK),    # K == 0
])
def test_bwd_dx_host_validation(args, code):
    assert _capi.lib().swiglu_bwd_dx(*args, None) == code


# swiglu_bwd_dw(dG, dU, X, dWg, dWu, M, K, N, dtype)
@pytest.mark.parametrize("args,code", [
    ((16, 32, 48, None, 80, 4, 64, 64, 0), _capi.SWIGLU_ERR_NULL_POINTER),
    ((16, None, 48, 1 << 20, 1 << 21, 4, 64, 64, 0), _capi.SWIGLU_ERR_NULL_POINTER),
    ((16, 32, 48, 1 << 20, (1 << 21) + 4, 4, 64, 64, 0), _capi.SWIGLU_ERR_MISALIGNED_PTR),
    ((16, 32, 48, 64, 80, 4, 64, 64, 2), _capi.SWIGLU_ERR_BAD_DTYPE),
    ((16, 32, 48, 64, 80, 4, 64, 12, 0), _capi.SWIGLU_ERR_MISALIGNED_DIM),
    ((16, 32, 48, 64, 80, 4, 64, 10, 1), _capi.SWIGLU_ERR_MISALIGNED_DIM),   # fp32: N % 4
    ((16, 32, 48, 64, 80, 4, -8, 64, 0), _capi.SWIGLU_ERR_BAD_DIM),
    # dWu [64,64] bf16 = 8 KiB starts inside dWg
    ((1 << 22, 1 << 23, 1 << 24, 1 << 20, (1 << 20) + 4096, 4, 64, 64, 0), _capi.SWIGLU_ERR_OVERLAP),
    # dWg on top of X
    ((1 << 22, 1 << 23, 1 << 20, 1 << 20, 1 << 24, 4, 64, 64, 0), _capi.SWIGLU_ERR_OVERLAP),
    ((None, None, None, None, None, 4, 64, 0, 0), _capi.SWIGLU_OK),    # N == 0
    ((None, None, None, None, None, 4, 0, 64, 0), _capi.SWIGLU_OK),    # K == 0
])
def test_bwd_dw_host_validation(args, code):
    assert _capi.lib().swiglu_bwd_dw(*args, None) == code


def test_bwd_gemm_no_device_is_an_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    lib = _capi.lib()
    assert lib.swiglu_bwd_dx(1 << 20, 1 << 21, 1 << 22, 1 << 23, 1 << 24, 4, 64, 64, 0,
                             None) == _capi.SWIGLU_ERR_NO_DEVICE
    # empty reduction still needs the device (it writes zeros)
    assert lib.swiglu_bwd_dw(None, None, None, 1 << 20, 1 << 21, 0, 64, 64, 0,
                             None) == _capi.SWIGLU_ERR_NO_DEVICE


def test_fwd_fp8_host_validation():
    import ctypes
    lib = _capi.lib()
    ok = (1 << 20, 1 << 21, 1 << 22, 1 << 23, 1 << 24)
    assert lib.swiglu_fwd_fp8(*ok, 4, 64, 40, None, None) == _capi.SWIGLU_ERR_MISALIGNED_DIM  # N % 16
    assert lib.swiglu_fwd_fp8(*ok, 4, 60, 64, None, None) == _capi.SWIGLU_ERR_MISALIGNED_DIM  # K % 8
    assert lib.swiglu_fwd_fp8(1 << 20, 1 << 21, 1 << 22, None, 1 << 24, 4, 64, 64, None,
                              None) == _capi.SWIGLU_ERR_NULL_POINTER
    assert lib.swiglu_fwd_fp8(1 << 20, 1 << 21, 1 << 22, (1 << 23) + 8, 1 << 24, 4, 64, 64, None,
                              None) == _capi.SWIGLU_ERR_MISALIGNED_PTR
    # scales may sit at any byte; Hq [4,64] bytes overlapping Hs
    assert lib.swiglu_fwd_fp8(1 << 20, 1 << 21, 1 << 22, 1 << 23, (1 << 23) + 255, 4, 64, 64,
                              None, None) == _capi.SWIGLU_ERR_OVERLAP
    with_gu = _capi.Epilogue(0, 1.0, 1 << 25, 1 << 26)
    assert lib.swiglu_fwd_fp8(*ok, 4, 64, 64, ctypes.byref(with_gu), None) == \
        _capi.SWIGLU_ERR_BAD_EPILOGUE
    assert lib.swiglu_fwd_fp8(None, None, None, None, None, 0, 64, 64, None, None) == _capi.SWIGLU_OK
