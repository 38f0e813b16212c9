"""A seeded sweep of random shapes through every route, forward and backward,
against the fp64 oracle on the whole output -- coverage beside the targeted
tests: decode (M <= 8), the tcgen05 weight stream (9 <= M <= 128 with K a
multiple of 64), the dual GEMM in its single-SM (M <= 128) and pair (M > 128)
forms, the fp32 3xTF32 GEMMs, and the backward GEMMs in both forms.  Shapes
are drawn from a fixed generator, so every run checks the same cases."""
import numpy as np
import pytest

import oracle
from gpu_util import assert_bf16_close, dev, f64, fp32_bound
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu


def _shapes(seed, count, m_bands, k_max, n_max):
    """(M, K, N) with K, N multiples of 8; M from the given bands in turn;
    every other shape with K a multiple of 64 (the weight stream's rule)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for i in range(count):
        lo, hi = m_bands[i % len(m_bands)]
        M = int(rng.integers(lo, hi + 1))
        K = 8 * int(rng.integers(1, k_max // 8 + 1))
        if i % 2 == 0:
            K = 64 * max(1, K // 64)
        N = 8 * int(rng.integers(1, n_max // 8 + 1))
        out.append((M, K, N))
    return out


FWD_BF16 = _shapes(1234, 36, [(1, 8), (9, 128), (129, 700)], 1100, 900)
FWD_F32 = _shapes(99, 9, [(1, 8), (9, 128), (129, 400)], 700, 600)
BWD = _shapes(4321, 12, [(1, 128), (129, 600)], 900, 700)


@pytest.mark.parametrize("M,K,N", FWD_BF16)
def test_sweep_forward_bf16(M, K, N):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 7 + K + N)
    H = _capi.swiglu_fwd(*(t.to(dev()) for t in (X, Wg, Wu)))
    assert _capi.swiglu_sync_status() == 0
    assert _capi.swiglu_last_route() == _capi.swiglu_route_for(M, K, N, _capi.SWIGLU_BF16)
    ref = oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"]
    assert_bf16_close(f64(H), ref, f"H {M}x{K}x{N}")


@pytest.mark.parametrize("M,K,N", FWD_F32)
def test_sweep_forward_fp32(M, K, N):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "f32", seed=M * 5 + K + N)
    H = _capi.swiglu_fwd(*(t.to(dev()) for t in (X, Wg, Wu)))
    assert _capi.swiglu_sync_status() == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_GEMM_TF32X3
    ref = oracle.swiglu_fwd(X, Wg, Wu, "f32", want_magnitudes=True)
    err = np.abs(f64(H) - ref["H"])
    bound = fp32_bound(ref["G"], ref["U"], ref["H"], ref["AG"], ref["AU"])
    assert np.all(err <= bound), float((err / bound).max())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,N", BWD)
def test_sweep_backward(dtype, M, K, N):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, dtype, seed=M * 3 + K + N)
    dG = synth.normal((M, N), N + 70, 1.0, dtype)
    dU = synth.normal((M, N), N + 71, 1.0, dtype)
    d = [t.to(dev()) for t in (dG, dU, Wg, Wu, X)]
    dX = _capi.swiglu_bwd_dx(d[0], d[1], d[2], d[3])
    dWg, dWu = _capi.swiglu_bwd_dw(d[0], d[1], d[4])
    assert _capi.swiglu_sync_status() == 0
    g, u, x, wg, wu = (f64(t) for t in (dG, dU, X, Wg, Wu))
    rdx = oracle.bwd_dx_f64(g, u, wg, wu)
    rg, ru = oracle.bwd_dw_f64(g, u, x)
    if dtype == "bf16":
        assert_bf16_close(f64(dX), rdx, f"dX {M}x{K}x{N}")
        assert_bf16_close(f64(dWg), rg, f"dWg {M}x{K}x{N}")
        assert_bf16_close(f64(dWu), ru, f"dWu {M}x{K}x{N}")
        return
    cases = ((dX, rdx, np.abs(g) @ np.abs(wg) + np.abs(u) @ np.abs(wu)),
             (dWg, rg, np.abs(g).T @ np.abs(x)), (dWu, ru, np.abs(u).T @ np.abs(x)))
    for got, r, mag in cases:
        e = np.abs(f64(got) - r)
        assert np.all(e <= 1e-5 * (mag + np.abs(r)) + 1e-30), float((e / (mag + 1e-30)).max())
