"""Epilogue variants (Liger-Kernel issue #937: swiglu/geglu activations and
the gate multiplier; TensorRT-LLM PR #17693: GELU(tanh) on the fp32
accumulator) and the training forward that also stores G and U, on every
route, against the fp64 oracle; and their backward."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (FP32_BWD_TOL, FP32_FWD_TOL, assert_bf16_close, assert_guards_intact,
                      assert_within, dev, f64, guarded_empty, to_dev)
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu

SILU, GELU = _capi.SWIGLU_ACT_SILU, _capi.SWIGLU_ACT_GELU_TANH


def _act_np(x, which):
    if which == GELU:
        return 0.5 * x * (1 + np.tanh(0.7978845608028654 * (x + 0.044715 * x ** 3)))
    return x / (1 + np.exp(-np.clip(x, -700, 700)))


def _arg_np(x, which):
    """The argument of the exponential in the kernel's evaluation: x for SiLU,
    2 c (x + a x^3) for GELU(tanh)."""
    if which == GELU:
        return 2 * 0.7978845608028654 * (x + 0.044715 * x ** 3)
    return x


def _dact_np(x, which):
    if which == GELU:
        y = 0.7978845608028654 * (x + 0.044715 * x ** 3)
        s = 1 / (1 + np.exp(-np.clip(2 * y, -700, 700)))
        return np.abs(s) + np.abs(2 * x * s * (1 - s) * 0.7978845608028654 * (1 + 3 * 0.044715 * x * x))
    s = 1 / (1 + np.exp(-np.clip(x, -700, 700)))
    return np.abs(s) * (1 + np.abs(x) * (1 - s))


def run_variant(X, Wg, Wu, which, alpha, store_gu):
    M, K = X.shape
    N = Wg.shape[0]
    Xd, Wgd, Wud = to_dev(X, Wg, Wu)
    fh, H = guarded_empty(M * N, X.dtype)
    epi_g = epi_u = None
    if store_gu:
        fg, Gb = guarded_empty(M * N, X.dtype)
        fu, Ub = guarded_empty(M * N, X.dtype)
        epi_g, epi_u = Gb, Ub
    import ctypes
    epi = _capi.Epilogue(which, alpha, epi_g.data_ptr() if store_gu else None,
                         epi_u.data_ptr() if store_gu else None)
    st = _capi.lib().swiglu_fwd_epilogue(Xd.data_ptr(), Wgd.data_ptr(), Wud.data_ptr(),
                                         H.data_ptr(), M, K, N,
                                         _capi._dtype_code(X), ctypes.byref(epi), 0,
                                         torch.cuda.current_stream().cuda_stream)
    assert st == 0, _capi.status_string(st)
    assert _capi.swiglu_sync_status() == 0
    assert_guards_intact(fh)
    out = {"H": H.view(M, N).cpu(), "route": _capi.swiglu_last_route()}
    if store_gu:
        assert_guards_intact(fg)
        assert_guards_intact(fu)
        out["G"] = epi_g.view(M, N).cpu()
        out["U"] = epi_u.view(M, N).cpu()
    return out


CASES = [  # (M, K, N, dtype, route)
    (1, 256, 512, "bf16", _capi.ROUTE_DECODE_BF16),
    (8, 1536, 1032, "bf16", _capi.ROUTE_DECODE_BF16),
    (24, 264, 72, "bf16", _capi.ROUTE_GEMM_BF16),
    (33, 1536, 1032, "bf16", _capi.ROUTE_STREAM_TC_BF16),
    (128, 256, 264, "bf16", _capi.ROUTE_STREAM_TC_BF16),
    (130, 192, 264, "bf16", _capi.ROUTE_GEMM_BF16),
    (300, 520, 392, "bf16", _capi.ROUTE_GEMM_BF16),
    (130, 96, 136, "f32", _capi.ROUTE_GEMM_TF32X3),
]


@pytest.mark.parametrize("M,K,N,dtype,route", CASES)
@pytest.mark.parametrize("which", [SILU, GELU])
@pytest.mark.parametrize("alpha", [1.0, 1.702, -0.5])
@pytest.mark.parametrize("store_gu", [False, True])
def test_forward_variants(M, K, N, dtype, route, which, alpha, store_gu):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, dtype, seed=M + K + which)
    out = run_variant(X, Wg, Wu, which, alpha, store_gu)
    assert out["route"] == route
    ref = oracle.swiglu_fwd(X, Wg, Wu, dtype, want_magnitudes=True, act=which, alpha=alpha)
    what = f"{dtype} M={M} act={which} alpha={alpha}"
    if dtype == "bf16":
        assert_bf16_close(f64(out["H"]), ref["H"], what)
        if store_gu:
            assert_bf16_close(f64(out["G"]), ref["G"], what + " G")
            assert_bf16_close(f64(out["U"]), ref["U"], what + " U")
    else:
        G, U = ref["G"], ref["U"]
        a = np.abs(alpha)
        bound = FP32_FWD_TOL * (np.abs(ref["H"]) + np.abs(_act_np(alpha * G, which)) * ref["AU"]
                                + np.abs(U) * a * _dact_np(alpha * G, which) * ref["AG"]) + 1e-30
        assert_within(np.abs(f64(out["H"]) - ref["H"]), bound, what)
        if store_gu:
            assert_within(np.abs(f64(out["G"]) - G), FP32_FWD_TOL * ref["AG"] + 1e-30, what + " G")
            assert_within(np.abs(f64(out["U"]) - U), FP32_FWD_TOL * ref["AU"] + 1e-30, what + " U")


def test_training_forward_integer_exact_gu():
    """Stored G and U are the fp32 accumulators rounded once to bf16: with
    integer operands G and U are exact in fp32, so the stored bits must be
    bf16_rne(G), bf16_rne(U) exactly, on every bf16 route."""
    for M, K, N in [(8, 256, 512), (256, 256, 384), (40, 256, 1032), (17, 200, 64)]:
        X, Wg, Wu = synth.integer_inputs(M, K, N, seed=M)
        out = run_variant(X, Wg, Wu, SILU, 1.0, True)
        G = (X.double() @ Wg.double().T).float().to(torch.bfloat16)
        U = (X.double() @ Wu.double().T).float().to(torch.bfloat16)
        assert torch.equal(out["G"].view(torch.int16), G.view(torch.int16)), M
        assert torch.equal(out["U"].view(torch.int16), U.view(torch.int16)), M


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("which", [SILU, GELU])
@pytest.mark.parametrize("alpha", [1.0, 1.702, -0.5])
def test_backward_variants(dtype, which, alpha):
    n = 100003
    dH, G, U = synth.dswiglu_inputs(n, dtype, seed=17 + which)
    dG, dU = _capi.dswiglu_bwd(*to_dev(dH, G, U), activation=which, gate_multiplier=alpha)
    assert _capi.swiglu_sync_status() == 0
    rG, rU = oracle.dswiglu(dH, G, U, dtype, act=which, alpha=alpha)
    what = f"bwd {dtype} act={which} alpha={alpha}"
    if dtype == "bf16":
        assert_bf16_close(f64(dG), rG, what + " dG")
        assert_bf16_close(f64(dU), rU, what + " dU")
    else:
        # The fp32 tolerance of the plain dSwiGLU (1e-6 of the terms), widened
        # by the conditioning of exp(z) when z itself carries rounding error:
        # for alpha != 1 or GELU the argument z = alpha g (resp. 2 c (x + a x^3))
        # is rounded, and exp multiplies its relative error by |z|.
        g, u, dh = f64(G), f64(U), f64(dH)
        z = np.abs(_arg_np(alpha * g, which))
        cond = 1.0 if (which == SILU and alpha == 1.0) else 1.0 + z
        bg = FP32_BWD_TOL * cond * (np.abs(rG) + np.abs(dh * u * alpha) * _dact_np(alpha * g, which)) + 1e-30
        bu = FP32_BWD_TOL * cond * (np.abs(rU) + np.abs(dh * alpha * g)) + 1e-30
        assert_within(np.abs(f64(dG) - rG), bg, what + " dG")
        assert_within(np.abs(f64(dU) - rU), bu, what + " dU")


def test_training_step_forward_then_backward():
    """A training step through the C ABI: the forward stores G and U, the
    backward consumes them -- checked against the oracle's backward on the
    same stored G and U, and against the oracle's own G and U."""
    M, K, N = 256, 512, 384
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=33)
    H, G, U = _capi.swiglu_fwd(*to_dev(X, Wg, Wu), return_gu=True, activation=GELU,
                               gate_multiplier=1.5)
    dH = synth.normal((M, N), 34, 1.0, "bf16")
    dG, dU = _capi.dswiglu_bwd(dH.to(dev()), G, U, activation=GELU, gate_multiplier=1.5)
    assert _capi.swiglu_sync_status() == 0
    rG, rU = oracle.dswiglu(dH, G.cpu(), U.cpu(), "bf16", act=GELU, alpha=1.5)
    assert_bf16_close(f64(dG), rG, "train dG")
    assert_bf16_close(f64(dU), rU, "train dU")
    ref = oracle.swiglu_fwd(X, Wg, Wu, "bf16", act=GELU, alpha=1.5)
    assert_bf16_close(f64(H), ref["H"], "train H")
    assert_bf16_close(f64(G), ref["G"], "train G")
