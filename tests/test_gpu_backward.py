"""Backward GEMMs of the projection (dX = dG Wg + dU Wu; dWg = dG^T X,
dWu = dU^T X -- the backward half of the fused MLP's forward/backward
dataflow, page "[RFC] Testing Methodology for FP32 Convergence Tests on
Fused SwiGLU/dSwiGLU Kernels", Background) through the C ABI, against the
fp64 oracle on the same bf16 inputs."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_bf16_close, assert_guards_intact, dev, f64, guarded_empty,
                      to_dev)
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu


def _grads(M, N, seed):
    return synth.normal((M, N), seed + 10), synth.normal((M, N), seed + 11)


def run_dx(dG, dU, Wg, Wu):
    M, N = dG.shape
    K = Wg.shape[1]
    dGd, dUd, Wgd, Wud = to_dev(dG, dU, Wg, Wu)
    full, dX = guarded_empty(M * K, torch.bfloat16)
    st = _capi.lib().swiglu_bwd_dx(dGd.data_ptr(), dUd.data_ptr(), Wgd.data_ptr(),
                                   Wud.data_ptr(), dX.data_ptr(), M, K, N, _capi.SWIGLU_BF16,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 0, _capi.status_string(st)
    assert _capi.swiglu_sync_status() == 0
    assert_guards_intact(full)
    return dX.view(M, K)


def run_dw(dG, dU, X):
    M, N = dG.shape
    K = X.shape[1]
    dGd, dUd, Xd = to_dev(dG, dU, X)
    fg, dWg = guarded_empty(N * K, torch.bfloat16)
    fu, dWu = guarded_empty(N * K, torch.bfloat16)
    st = _capi.lib().swiglu_bwd_dw(dGd.data_ptr(), dUd.data_ptr(), Xd.data_ptr(),
                                   dWg.data_ptr(), dWu.data_ptr(), M, K, N, _capi.SWIGLU_BF16,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 0, _capi.status_string(st)
    assert _capi.swiglu_sync_status() == 0
    assert_guards_intact(fg)
    assert_guards_intact(fu)
    return dWg.view(N, K), dWu.view(N, K)


# (M, K, N): single tile, ragged tails in every dimension (K not a multiple of
# 64, N not a multiple of 64 or 128), several tiles each way.  dX takes the
# pair form (256-row tiles over two SMs) where M > 128 and dW where N > 128,
# else one SM per tile.  With 148 SMs (74 pairs) the tile-width model picks:
# pairs 256 wide for dX of (1300, 2560, 136) and (4800, 448, 72) and dW of
# (200, 2048, 1032) and (100, 448, 2376), pairs 128 wide for dX and dW of
# (130, 264, 200) and (300, 520, 136); single SMs 128 wide for the small-M dX
# and small-N dW, 192 wide for dW of (64, 9600, 104).  M = 257 and N = 1544
# leave the odd CTA of the last pair wholly outside the matrix.
SHAPES = [(1, 8, 8), (130, 264, 200), (300, 520, 136), (257, 1032, 72), (64, 128, 64),
          (1300, 2560, 136), (200, 2048, 1032), (9, 64, 1544), (4800, 448, 72),
          (100, 448, 2376), (64, 9600, 104)]


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_bwd_dx_matches_oracle(M, K, N):
    _, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=M + K)
    dG, dU = _grads(M, N, seed=N)
    dX = run_dx(dG, dU, Wg, Wu)
    assert _capi.swiglu_last_route() == _capi.ROUTE_BWD_GEMM_BF16
    ref = oracle.bwd_dx_f64(f64(dG), f64(dU), f64(Wg), f64(Wu))
    assert_bf16_close(f64(dX), ref, f"dX {M}x{K}x{N}")


@pytest.mark.parametrize("M,K,N", SHAPES)
def test_bwd_dw_matches_oracle(M, K, N):
    X, _, _ = synth.swiglu_inputs(M, K, N, seed=M + K)
    dG, dU = _grads(M, N, seed=N)
    dWg, dWu = run_dw(dG, dU, X)
    assert _capi.swiglu_last_route() == _capi.ROUTE_BWD_GEMM_BF16
    rg, ru = oracle.bwd_dw_f64(f64(dG), f64(dU), f64(X))
    assert_bf16_close(f64(dWg), rg, f"dWg {M}x{K}x{N}")
    assert_bf16_close(f64(dWu), ru, f"dWu {M}x{K}x{N}")


@pytest.mark.parametrize("M,K,N", [(300, 264, 200), (130, 1032, 1544), (1300, 2560, 136)])
def test_bwd_integer_exact(M, K, N):
    """Ternary operands: every sum is a small integer, exact in fp32 in any
    order and, below 256 in magnitude, exact in bf16 -- so the outputs must
    match the oracle bit for bit (a wrong index, operand or tail fails)."""
    X = synth.ternary((M, K), 1, 0.5)
    Wg = synth.ternary((N, K), 2, 0.05)
    Wu = synth.ternary((N, K), 3, 0.05)
    dG = synth.ternary((M, N), 4, 0.05)
    dU = synth.ternary((M, N), 5, 0.05)
    rdx = oracle.bwd_dx_f64(f64(dG), f64(dU), f64(Wg), f64(Wu))
    rg, ru = oracle.bwd_dw_f64(f64(dG), f64(dU), f64(X))
    for r in (rdx, rg, ru):
        assert np.abs(r).max() <= 256 and np.abs(r).max() >= 2
    np.testing.assert_array_equal(f64(run_dx(dG, dU, Wg, Wu)), rdx)
    dWg, dWu = run_dw(dG, dU, X)
    np.testing.assert_array_equal(f64(dWg), rg)
    np.testing.assert_array_equal(f64(dWu), ru)


def test_bwd_pairs_are_not_swapped():
    """dU = 0: dX must equal dG Wg alone (and dWu must be exactly zero)."""
    M, K, N = 200, 264, 136
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=5)
    dG, _ = _grads(M, N, seed=7)
    dU = torch.zeros_like(dG)
    dX = run_dx(dG, dU, Wg, Wu)
    assert_bf16_close(f64(dX), f64(dG) @ f64(Wg), "dX with dU = 0")
    dWg, dWu = run_dw(dG, dU, X)
    assert not bool(dWu.any())
    assert_bf16_close(f64(dWg), f64(dG).T @ f64(X), "dWg")


def test_bwd_empty_and_degenerate():
    s = torch.cuda.current_stream().cuda_stream
    lib = _capi.lib()
    # N == 0: dX = 0 (the empty reduction), dW untouched-and-empty.
    full, dX = guarded_empty(5 * 64, torch.bfloat16)
    assert lib.swiglu_bwd_dx(None, None, None, None, dX.data_ptr(), 5, 64, 0, 0, s) == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_ZERO_K
    torch.cuda.synchronize()
    assert not bool(dX.any()) and not bool(torch.signbit(dX).any())
    assert_guards_intact(full)
    # M == 0: dWg = dWu = 0.
    fg, dWg = guarded_empty(16 * 64, torch.bfloat16)
    fu, dWu = guarded_empty(16 * 64, torch.bfloat16)
    assert lib.swiglu_bwd_dw(None, None, None, dWg.data_ptr(), dWu.data_ptr(), 0, 64, 16, 0,
                             s) == 0
    torch.cuda.synchronize()
    assert not bool(dWg.any()) and not bool(dWu.any())
    assert_guards_intact(fg)
    assert_guards_intact(fu)
    # M == 0 for dX / N == 0 for dW: nothing to write, nothing enqueued.
    assert lib.swiglu_bwd_dx(None, None, None, None, None, 0, 64, 64, 0, s) == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_NONE
    assert lib.swiglu_bwd_dw(None, None, None, None, None, 7, 64, 0, 0, s) == 0


def test_bwd_deterministic():
    M, K, N = 520, 1032, 264
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=3)
    dG, dU = _grads(M, N, seed=4)
    a = run_dx(dG, dU, Wg, Wu).clone()
    b = run_dx(dG, dU, Wg, Wu)
    assert torch.equal(a, b)
    g1, u1 = run_dw(dG, dU, X)
    g1, u1 = g1.clone(), u1.clone()
    g2, u2 = run_dw(dG, dU, X)
    assert torch.equal(g1, g2) and torch.equal(u1, u2)


def test_bwd_python_binding_shapes():
    M, K, N = 3 * 70, 264, 136
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=9)
    dG, dU = _grads(M, N, seed=9)
    Xd, Wgd, Wud, dGd, dUd = to_dev(X, Wg, Wu, dG, dU)
    dX = _capi.swiglu_bwd_dx(dGd.view(3, 70, N), dUd.view(3, 70, N), Wgd, Wud)
    assert dX.shape == (3, 70, K)
    dWg, dWu = _capi.swiglu_bwd_dw(dGd.view(3, 70, N), dUd.view(3, 70, N), Xd.view(3, 70, K))
    assert dWg.shape == (N, K) and dWu.shape == (N, K)
    assert_bf16_close(f64(dX).reshape(M, K), oracle.bwd_dx_f64(f64(dG), f64(dU), f64(Wg), f64(Wu)),
                      "dX via binding")
    with pytest.raises(TypeError):   # mixed dtypes
        _capi.swiglu_bwd_dx(dGd, dUd, Wgd.float(), Wud.float())
    # N == 0 through the binding: dX = 0 (empty reduction), dW empty
    e = torch.empty((5, 0), dtype=torch.bfloat16, device=dev())
    w = torch.empty((0, 64), dtype=torch.bfloat16, device=dev())
    dX0 = _capi.swiglu_bwd_dx(e, e, w, w)
    torch.cuda.synchronize()
    assert dX0.shape == (5, 64) and not bool(dX0.any())


def test_training_step_full_size_sampled():
    """The whole training step at the prefill size (M=4096 tokens, K=4096,
    N=14336): forward storing G and U, dSwiGLU, dX and dW -- each stage
    checked on sampled outputs against the oracle fed that stage's GPU
    inputs."""
    M, K, N = 4096, 4096, 14336
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=21)
    dH = synth.normal((M, N), 22)
    Xd, Wgd, Wud, dHd = to_dev(X, Wg, Wu, dH)
    H, G, U = _capi.swiglu_fwd(Xd, Wgd, Wud, return_gu=True)
    dG, dU = _capi.dswiglu_bwd(dHd, G, U)
    dX = _capi.swiglu_bwd_dx(dG, dU, Wgd, Wud)
    dWg, dWu = _capi.swiglu_bwd_dw(dG, dU, Xd)
    assert _capi.swiglu_sync_status() == 0
    r = np.random.Generator(np.random.PCG64(5))
    rows = np.concatenate([r.integers(0, M, 6), [0, M - 1]])
    cols = np.concatenate([r.integers(0, N, 6), [0, N - 1]])
    dGc, dUc = dG.cpu(), dU.cpu()
    ref_dx = oracle.bwd_dx_f64(f64(dGc[rows]), f64(dUc[rows]), f64(Wg), f64(Wu))
    assert_bf16_close(f64(dX.cpu()[rows]), ref_dx, "dX rows (full size)")
    rg, ru = oracle.bwd_dw_f64(f64(dGc[:, cols]), f64(dUc[:, cols]), f64(X))
    assert_bf16_close(f64(dWg.cpu()[cols]), rg, "dWg rows (full size)")
    assert_bf16_close(f64(dWu.cpu()[cols]), ru, "dWu rows (full size)")
    rdg, rdu = oracle.dswiglu_f64(f64(dH[rows]), f64(G.cpu()[rows]), f64(U.cpu()[rows]))
    assert_bf16_close(f64(dGc[rows]), rdg, "dG rows")
    assert_bf16_close(f64(dUc[rows]), rdu, "dU rows")


# ---- fp32 (3xTF32) -----------------------------------------------------------

def _run_f32(fn, *args):
    out = fn(*(a.to(dev()) for a in args))
    assert _capi.swiglu_sync_status() == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_BWD_GEMM_TF32X3
    return out


# With 148 SMs, dX alone (the cost model of the split tail) takes 128-wide
# tiles with the tail split 2 ways for (130, 260, 196) and (300, 516, 136)
# and 19 ways for (100, 448, 2376), 256-wide ones split 9 ways for
# (200, 2048, 1032), and unsplit 192-wide ones for (4800, 448, 72); dW takes
# 192-wide tiles for (100, 448, 2376), 256-wide ones for (200, 2048, 1032)
# and 128-wide ones elsewhere.
@pytest.mark.parametrize("M,K,N", [(1, 4, 4), (130, 260, 196), (300, 516, 136), (257, 1028, 68),
                                   (200, 2048, 1032), (4800, 448, 72), (100, 448, 2376)])
def test_bwd_fp32_within_mixed_bound(M, K, N):
    """fp32 backward GEMMs within 1e-5 of the size of the terms summed
    (sum |dG||Wg| + |dU||Wu|, resp. sum |dG||X|): the fp32 forward's bound,
    read the same way for the backward."""
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "f32", seed=M + 1)
    dG = synth.normal((M, N), N + 20, 1.0, "f32")
    dU = synth.normal((M, N), N + 21, 1.0, "f32")
    g, u, x, wg, wu = (f64(t) for t in (dG, dU, X, Wg, Wu))
    dX = _run_f32(_capi.swiglu_bwd_dx, dG, dU, Wg, Wu)
    ref = oracle.bwd_dx_f64(g, u, wg, wu)
    mag = np.abs(g) @ np.abs(wg) + np.abs(u) @ np.abs(wu)
    err = np.abs(f64(dX) - ref)
    assert np.all(err <= 1e-5 * (mag + np.abs(ref)) + 1e-30), float((err / (mag + 1e-30)).max())
    dWg, dWu = _run_f32(_capi.swiglu_bwd_dw, dG, dU, X)
    rg, ru = oracle.bwd_dw_f64(g, u, x)
    for got, r, mg in ((dWg, rg, np.abs(g).T @ np.abs(x)), (dWu, ru, np.abs(u).T @ np.abs(x))):
        e = np.abs(f64(got) - r)
        assert np.all(e <= 1e-5 * (mg + np.abs(r)) + 1e-30), float((e / (mg + 1e-30)).max())
    # near-IEEE: norm-wise error well below plain TF32's (~1e-4 at these sizes)
    assert np.linalg.norm(f64(dX) - ref) <= 1e-5 * np.linalg.norm(ref)


def test_bwd_fp32_integer_exact():
    """Small integers are exact in TF32's hi part (lo = 0) and every sum is
    exact in fp32: bit-exact against the oracle."""
    M, K, N = 300, 264, 200
    X = synth.ternary((M, K), 1, 0.5, "f32")
    Wg = synth.ternary((N, K), 2, 0.05, "f32")
    Wu = synth.ternary((N, K), 3, 0.05, "f32")
    dG = synth.ternary((M, N), 4, 0.05, "f32")
    dU = synth.ternary((M, N), 5, 0.05, "f32")
    np.testing.assert_array_equal(f64(_run_f32(_capi.swiglu_bwd_dx, dG, dU, Wg, Wu)),
                                  oracle.bwd_dx_f64(f64(dG), f64(dU), f64(Wg), f64(Wu)))
    dWg, dWu = _run_f32(_capi.swiglu_bwd_dw, dG, dU, X)
    rg, ru = oracle.bwd_dw_f64(f64(dG), f64(dU), f64(X))
    np.testing.assert_array_equal(f64(dWg), rg)
    np.testing.assert_array_equal(f64(dWu), ru)


# dX alone with the split tail (148 SMs: 1280 x 4096 has 160 tiles of 256
# columns, 12 beyond the first wave, split 8 ways; 256 x 512 has 4 tiles of
# 128, split 16 ways; 300 x 520 has 9, split 2 ways).
@pytest.mark.parametrize("M,K,N,rows", [(1280, 4096, 1024, "sampled"), (256, 512, 2048, "all"),
                                        (300, 520, 200, "all")])
def test_bwd_fp32_split_tail(M, K, N, rows):
    """dX alone, where the last partial wave of tiles is split along the
    reduction and the parts' partial sums are added in a fixed order:
    within the mixed bound of the oracle (sampled rows from every 128-row
    block, or all rows) and bitwise identical on a second call."""
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "f32", seed=M + 5)
    dG = synth.normal((M, N), N + 40, 1.0, "f32")
    dU = synth.normal((M, N), N + 41, 1.0, "f32")
    d = [t.to(dev()) for t in (dG, dU, Wg, Wu)]
    dX = _run_f32(_capi.swiglu_bwd_dx, *d)
    again = _run_f32(_capi.swiglu_bwd_dx, *d)
    assert torch.equal(dX, again)
    if rows == "all":
        r = np.arange(M)
    else:
        r = np.unique(np.concatenate([np.arange(0, M, 128) + o for o in (0, 61, 127)]))
        r = r[r < M]
    g, u, wg, wu = f64(dG)[r], f64(dU)[r], f64(Wg), f64(Wu)
    ref = oracle.bwd_dx_f64(g, u, wg, wu)
    mag = np.abs(g) @ np.abs(wg) + np.abs(u) @ np.abs(wu)
    err = np.abs(f64(dX)[r] - ref)
    assert np.all(err <= 1e-5 * (mag + np.abs(ref)) + 1e-30), float((err / (mag + 1e-30)).max())
    assert np.linalg.norm(f64(dX)[r] - ref) <= 1e-5 * np.linalg.norm(ref)


def test_bwd_fp32_split_tail_in_cuda_graph():
    """fp32 dX alone with its split tail -- whose workspace is allocated and
    freed in stream order inside the call -- captured in a CUDA graph: two
    replays give the eager call's bits."""
    M, K, N = 1280, 4096, 1024
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "f32", seed=M + 7)
    dG = synth.normal((M, N), N + 42, 1.0, "f32")
    dU = synth.normal((M, N), N + 43, 1.0, "f32")
    d = [t.to(dev()) for t in (dG, dU, Wg, Wu)]
    ref = _run_f32(_capi.swiglu_bwd_dx, *d)
    s = torch.cuda.Stream()
    out = torch.empty_like(ref)
    with torch.cuda.stream(s):
        _capi.swiglu_bwd_dx(*d, dX=out, stream=s)   # warm-up outside the capture
    torch.cuda.synchronize()
    out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        _capi.swiglu_bwd_dx(*d, dX=out, stream=s)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        assert _capi.swiglu_sync_status() == 0
        assert torch.equal(out, ref)
    del g


def test_bwd_fp32_split_tail_two_streams():
    """Two fp32 dX calls with split tails on two streams at once: each takes
    its own workspace from the pool in its stream's order, so both give the
    bits of the same calls made one after the other."""
    M, K, N = 1280, 4096, 1024
    ins = []
    for s in (0, 1):
        X, Wg, Wu = synth.swiglu_inputs(M, K, N, "f32", seed=M + 20 + s)
        dG = synth.normal((M, N), N + 50 + s, 1.0, "f32")
        dU = synth.normal((M, N), N + 60 + s, 1.0, "f32")
        ins.append([t.to(dev()) for t in (dG, dU, Wg, Wu)])
    refs = [_run_f32(_capi.swiglu_bwd_dx, *d) for d in ins]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    outs = [torch.empty_like(r) for r in refs]
    torch.cuda.synchronize()
    for _ in range(3):
        for d, o, s in zip(ins, outs, streams):
            _capi.swiglu_bwd_dx(*d, dX=o, stream=s)
    torch.cuda.synchronize()
    assert _capi.swiglu_sync_status() == 0
    for o, r in zip(outs, refs):
        assert torch.equal(o, r)


def test_bwd_fp32_split_tail_integer_exact():
    """Integer operands with exact fp32 sums: every part's partial sum and
    their total are exact, so dX alone with a split tail equals the oracle
    bit for bit (sampled rows from every 128-row block)."""
    M, K, N = 1280, 4096, 1024
    Wg = synth.ternary((N, K), 12, 0.05, "f32")
    Wu = synth.ternary((N, K), 13, 0.05, "f32")
    dG = synth.ternary((M, N), 14, 0.05, "f32")
    dU = synth.ternary((M, N), 15, 0.05, "f32")
    dX = f64(_run_f32(_capi.swiglu_bwd_dx, dG, dU, Wg, Wu))
    r = np.concatenate([np.arange(0, M, 128) + o for o in (0, 77, 127)])
    np.testing.assert_array_equal(dX[r], oracle.bwd_dx_f64(f64(dG)[r], f64(dU)[r], f64(Wg),
                                                           f64(Wu)))


def test_bwd_fp32_full_size_sampled():
    """LLaMA-2 13B fp32 shape at M = 2048 (the fp32 forward's workload):
    sampled rows of dX and of dWg, dWu against the oracle, mixed bound."""
    M, K, N = 2048, 5120, 13824
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "f32", seed=77)
    dG = synth.normal((M, N), 78, 1.0, "f32")
    dU = synth.normal((M, N), 79, 1.0, "f32")
    dX = _run_f32(_capi.swiglu_bwd_dx, dG, dU, Wg, Wu).cpu()
    dWg, dWu = _run_f32(_capi.swiglu_bwd_dw, dG, dU, X)
    dWg, dWu = dWg.cpu(), dWu.cpu()
    rows = np.array([0, 1, 1000, 2047])
    cols = np.array([0, 5000, 13823])
    g, u, wg, wu, x = f64(dG), f64(dU), f64(Wg), f64(Wu), f64(X)
    ref = oracle.bwd_dx_f64(g[rows], u[rows], wg, wu)
    mag = np.abs(g[rows]) @ np.abs(wg) + np.abs(u[rows]) @ np.abs(wu)
    assert np.all(np.abs(f64(dX)[rows] - ref) <= 1e-5 * mag + 1e-30)
    rg, ru = oracle.bwd_dw_f64(g[:, cols], u[:, cols], x)
    assert np.all(np.abs(f64(dWg)[cols] - rg) <= 1e-5 * (np.abs(g[:, cols]).T @ np.abs(x)) + 1e-30)
    assert np.all(np.abs(f64(dWu)[cols] - ru) <= 1e-5 * (np.abs(u[:, cols]).T @ np.abs(x)) + 1e-30)


# ---- all three GEMMs in one call -------------------------------------------

@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("M,K,N", [(130, 264, 200), (257, 1032, 72), (2048, 520, 264),
                                   (1, 8, 8)])
def test_bwd_gemms_equals_separate_calls(dtype, M, K, N):
    """swiglu_bwd_gemms gives exactly the separate calls' results (for fp32 it
    is one scheduled launch; every tile's arithmetic is the same) and matches
    the oracle -- except fp32 dX where the separate dX call splits its tail
    tiles along the reduction (sums in another order): there both are held
    to the oracle's bound instead."""
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, dtype, seed=M + 3)
    dG = synth.normal((M, N), N + 30, 1.0, dtype)
    dU = synth.normal((M, N), N + 31, 1.0, dtype)
    d = to_dev(dG, dU, Wg, Wu, X)
    dX, dWg, dWu = _capi.swiglu_bwd_gemms(*d)
    assert _capi.swiglu_sync_status() == 0
    sx = _capi.swiglu_bwd_dx(d[0], d[1], d[2], d[3])
    sg, su = _capi.swiglu_bwd_dw(d[0], d[1], d[4])
    assert _capi.swiglu_sync_status() == 0
    assert torch.equal(dWg, sg) and torch.equal(dWu, su)
    if dtype == "f32":
        g, u = f64(dG), f64(dU)
        ref = oracle.bwd_dx_f64(g, u, f64(Wg), f64(Wu))
        mag = np.abs(g) @ np.abs(f64(Wg)) + np.abs(u) @ np.abs(f64(Wu))
        for got in (dX, sx):
            assert np.all(np.abs(f64(got) - ref) <= 1e-5 * (mag + np.abs(ref)) + 1e-30)
    else:
        assert torch.equal(dX, sx)
        assert_bf16_close(f64(dX), oracle.bwd_dx_f64(f64(dG), f64(dU), f64(Wg), f64(Wu)), "dX")
        rg, ru = oracle.bwd_dw_f64(f64(dG), f64(dU), f64(X))
        assert_bf16_close(f64(dWg), rg, "dWg")
        assert_bf16_close(f64(dWu), ru, "dWu")


def test_bwd_gemms_fp32_integer_exact_13b_schedule():
    """The schedule of the 13B shape at M = 2048 (320 dX tiles, 2.2 waves, and
    4320 dW tiles) on integer operands: bit-exact against the oracle on
    sampled rows -- every tile is computed once and stored where it belongs."""
    M, K, N = 2048, 5120, 13824
    X = synth.ternary((M, K), 1, 0.5, "f32")
    Wg = synth.ternary((N, K), 2, 0.02, "f32")
    Wu = synth.ternary((N, K), 3, 0.02, "f32")
    dG = synth.ternary((M, N), 4, 0.02, "f32")
    dU = synth.ternary((M, N), 5, 0.02, "f32")
    dX, dWg, dWu = _capi.swiglu_bwd_gemms(*to_dev(dG, dU, Wg, Wu, X))
    assert _capi.swiglu_sync_status() == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_BWD_GEMM_TF32X3
    r = np.random.Generator(np.random.PCG64(8))
    rows = np.concatenate([r.integers(0, M, 5), [0, 127, 128, M - 1]])
    cols = np.concatenate([r.integers(0, N, 5), [0, 127, 128, N - 1]])
    g, u = f64(dG), f64(dU)
    np.testing.assert_array_equal(f64(dX.cpu())[rows],
                                  oracle.bwd_dx_f64(g[rows], u[rows], f64(Wg), f64(Wu)))
    rg, ru = oracle.bwd_dw_f64(g[:, cols], u[:, cols], f64(X))
    np.testing.assert_array_equal(f64(dWg.cpu())[cols], rg)
    np.testing.assert_array_equal(f64(dWu.cpu())[cols], ru)
