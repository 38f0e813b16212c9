"""dSwiGLU kernel vs the fp64 oracle (bf16 and fp32), through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (FP32_BWD_TOL, assert_bf16_close, assert_guards_intact, assert_within, dev,
                      f64, guarded_empty, to_dev)
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu


def _run(dH, G, U):
    dHd, Gd, Ud = to_dev(dH, G, U)
    fg, dG = guarded_empty(G.numel(), G.dtype)
    fu, dU = guarded_empty(G.numel(), G.dtype)
    _capi.dswiglu_bwd(dHd, Gd, Ud, dG, dU)
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert_guards_intact(fg)
    assert_guards_intact(fu)
    return dG.cpu(), dU.cpu()


def _fp32_bounds(dh, g, u, dG_ref, dU_ref):
    """1e-6 of the magnitudes of the terms before cancellation:
    dG: |dG| + |dh u s| + |dh u s g (1-s)|;  dU: |dU| with floor |dh g s|."""
    s = 1.0 / (1.0 + np.exp(-np.clip(g, -700, 700)))
    bg = FP32_BWD_TOL * (np.abs(dG_ref) + np.abs(dh * u * s) + np.abs(dh * u * s * g * (1 - s))) + 1e-30
    bu = FP32_BWD_TOL * (np.abs(dU_ref) + np.abs(dh * g * s)) + 1e-30
    return bg, bu


@pytest.mark.parametrize("n", [1, 7, 8, 9, 2048, 4095, 1000003])
def test_dswiglu_bf16_ragged(n):
    dH, G, U = synth.dswiglu_inputs(n, "bf16", seed=n)
    dG, dU = _run(dH, G, U)
    rG, rU = oracle.dswiglu(dH, G, U, "bf16")
    assert_bf16_close(f64(dG), rG, f"dG n={n}")
    assert_bf16_close(f64(dU), rU, f"dU n={n}")


@pytest.mark.parametrize("n", [1, 3, 4, 5, 2048, 1000003])
def test_dswiglu_fp32_ragged(n):
    dH, G, U = synth.dswiglu_inputs(n, "f32", seed=n)
    dG, dU = _run(dH, G, U)
    rG, rU = oracle.dswiglu(dH, G, U, "f32")
    bg, bu = _fp32_bounds(f64(dH), f64(G), f64(U), rG, rU)
    assert_within(np.abs(f64(dG) - rG), bg, f"fp32 dG n={n}")
    assert_within(np.abs(f64(dU) - rU), bu, f"fp32 dU n={n}")


def test_dswiglu_tiny_from_forward():
    """Tiny config: G, U are the oracle's forward G, U for X[4,256], W[512,256]
    (seed 0), rounded to bf16; dH ~ N(0,1) from its own seed."""
    X, Wg, Wu = synth.swiglu_inputs(4, 256, 512, "bf16", seed=0)
    fwd = oracle.swiglu_fwd(X, Wg, Wu, "bf16")
    G = torch.from_numpy(fwd["G"]).to(torch.bfloat16).reshape(-1)
    U = torch.from_numpy(fwd["U"]).to(torch.bfloat16).reshape(-1)
    dH = synth.normal((G.numel(),), 3, 1.0, "bf16")
    dG, dU = _run(dH, G, U)
    rG, rU = oracle.dswiglu(dH, G, U, "bf16")
    assert_bf16_close(f64(dG), rG, "tiny dG")
    assert_bf16_close(f64(dU), rU, "tiny dU")


def test_dswiglu_special_values():
    """g = 0, +-large, the silu minimum, dh = 0, u = 0, and non-finite inputs
    (NaN/Inf propagate as IEEE arithmetic says)."""
    g = torch.tensor([0.0, 40.0, -40.0, -1.2784645, 3.0, 2.0, float("nan"), 1.0, -90.0, 90.0],
                     dtype=torch.float32)
    u = torch.tensor([3.0, 2.0, 2.0, 1.5, 0.0, 1.0, 1.0, float("inf"), 1.0, 1.0])
    dh = torch.tensor([2.0, 1.0, 1.0, 1.0, 1.0, 0.0, 1.0, 1.0, 1.0, 1.0])
    for dtype in ("bf16", "f32"):
        tdt = synth.DTYPES[dtype]
        dG, dU = _run(dh.to(tdt), g.to(tdt), u.to(tdt))
        rG, rU = oracle.dswiglu(dh.to(tdt), g.to(tdt), u.to(tdt), dtype)
        gG, gU = f64(dG), f64(dU)
        for arr_gpu, arr_ref, name in ((gG, rG, "dG"), (gU, rU, "dU")):
            fin = np.isfinite(arr_ref)
            assert np.array_equal(np.isnan(arr_gpu), np.isnan(arr_ref)), (dtype, name)
            assert np.array_equal(np.isinf(arr_gpu), np.isinf(arr_ref)), (dtype, name)
            if dtype == "bf16":
                assert_bf16_close(arr_gpu[fin], arr_ref[fin], f"special {name}")
        if dtype == "f32":
            fin = np.isfinite(rG) & np.isfinite(rU)
            bg, bu = _fp32_bounds(f64(dh)[fin], f64(g)[fin], f64(u)[fin], rG[fin], rU[fin])
            assert_within(np.abs(gG[fin] - rG[fin]), bg, "special fp32 dG")
            assert_within(np.abs(gU[fin] - rU[fin]), bu, "special fp32 dU")


def test_dswiglu_in_place():
    n = 10007
    dH, G, U = synth.dswiglu_inputs(n, "bf16", seed=5)
    rG, rU = oracle.dswiglu(dH, G, U, "bf16")
    dHd, Gd, Ud = to_dev(dH, G, U)
    _capi.dswiglu_bwd(dHd, Gd, Ud, Gd, Ud)  # dG -> G, dU -> U
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert_bf16_close(f64(Gd), rG, "in-place dG")
    assert_bf16_close(f64(Ud), rU, "in-place dU")


def test_dswiglu_full_size_sampled():
    """Prefill-backward config: n = 8192 * 14336 bf16, the launch the bench
    times; checked on sampled elements plus the first/last vectors."""
    n = 8192 * 14336
    dH, G, U = synth.dswiglu_inputs(n, "bf16", seed=0)
    dG, dU = _run(dH, G, U)
    r = np.random.Generator(np.random.PCG64(99))
    idx = np.concatenate([r.integers(0, n, size=200000), np.arange(16), np.arange(n - 16, n)])
    rG, rU = oracle.dswiglu(dH[idx], G[idx], U[idx], "bf16")
    assert_bf16_close(f64(dG[idx]), rG, "full dG")
    assert_bf16_close(f64(dU[idx]), rU, "full dU")
    # deterministic: a second run is bitwise identical
    dG2, dU2 = _run(dH, G, U)
    assert torch.equal(dG.view(torch.int16), dG2.view(torch.int16))
    assert torch.equal(dU.view(torch.int16), dU2.view(torch.int16))
