"""Quantised output (fp8 e4m3 H with UE8M0 scales per (1,32) block, the
e4m3 output and sf_block = (1,32) scale factors of TileKernels-PTO PR #20)
through the C ABI, against the oracle's quantisation of its fp64 H."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import dev, f64, to_dev
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu

GELU = _capi.SWIGLU_ACT_GELU_TANH


def _dec(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, dtype=np.uint8))
    return t.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def run(X, Wg, Wu, act=0, alpha=1.0):
    Hq, Hs = _capi.swiglu_fwd_fp8(*to_dev(X, Wg, Wu), activation=act, gate_multiplier=alpha)
    assert _capi.swiglu_sync_status() == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_GEMM_BF16
    return Hq.cpu().numpy(), Hs.cpu().numpy()


@pytest.mark.parametrize("M,K,N", [(130, 256, 272), (8, 128, 64), (1, 64, 16), (300, 256, 400)])
def test_fp8_integer_exact(M, K, N):
    """Integer operands with every gate >= 17: h = G U exactly in fp32 and
    in the oracle, so the scale codes and e4m3 codes must match bit for bit
    (ragged 32-column blocks and row/column tails included)."""
    X, Wg, Wu = synth.integer_inputs(M, K, N)
    q, s = run(X, Wg, Wu)
    ref = oracle.swiglu_fwd_f64(f64(X), f64(Wg), f64(Wu))["H"]
    rq, rs = oracle.quant_e4m3(ref)
    np.testing.assert_array_equal(s, rs)
    np.testing.assert_array_equal(q, rq)


def _check_close(q, s, H):
    """Scale codes equal unless amax sits within 1e-4 of a power-of-two
    boundary; codes equal unless h / 2^e sits within 2e-3 (relative, plus
    2^-10 absolute: a quarter of the smallest half-step at |x| >= 2^-4) of a
    midpoint between two e4m3 values, and then they are neighbours.  The
    kernel quantises its fp32 h, the oracle the fp64 one: only decisions
    within that rounding distance may differ."""
    rq, rs = oracle.quant_e4m3(H)
    M, N = H.shape
    nb = rs.shape[1]
    amax = np.zeros((M, nb))
    for b in range(nb):
        amax[:, b] = np.abs(H[:, 32 * b:32 * b + 32]).max(axis=1)
    scale_diff = s.astype(int) != rs.astype(int)
    if scale_diff.any():
        e = rs.astype(int) - 127
        ratio = amax / (448.0 * 2.0 ** e)      # in (0.5, 1]
        near = (np.abs(ratio - 1.0) < 1e-4) | (np.abs(ratio - 0.5) < 1e-4)
        assert np.all(near[scale_diff]), "scale codes differ away from a boundary"
        assert np.all(np.abs(s.astype(int) - rs.astype(int))[scale_diff] == 1)
    e_full = np.repeat(s.astype(int) - 127, 32, axis=1)[:, :N]
    same_scale = np.repeat(~scale_diff, 32, axis=1)[:, :N]
    vg, vr = _dec(q), _dec(rq)
    diff = (q != rq) & same_scale
    if diff.any():
        x = (H * 2.0 ** -e_full)[diff]
        lo, hi = np.minimum(vg[diff], vr[diff]), np.maximum(vg[diff], vr[diff])
        mid = (lo + hi) / 2
        assert np.all(np.abs(np.abs(x) - np.abs(mid)) <= 2e-3 * np.abs(x) + 2.0 ** -10), \
            "codes differ away from a rounding midpoint"
        # neighbours on the e4m3 grid: no representable value strictly between
        grid = np.unique(np.abs(_dec(np.arange(127))))
        between = [np.sum((grid > a) & (grid < b)) for a, b in zip(np.abs(lo), np.abs(hi))]
        assert max(between) == 0
    return int(diff.sum()), int(scale_diff.sum())


@pytest.mark.parametrize("M,K,N,act,alpha", [(257, 512, 400, 0, 1.0), (64, 1024, 1024, GELU, 1.5),
                                             (5, 256, 272, 0, -0.7)])
def test_fp8_matches_oracle(M, K, N, act, alpha):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=M)
    q, s = run(X, Wg, Wu, act, alpha)
    ref = oracle.swiglu_fwd_f64(f64(X), f64(Wg), f64(Wu), act=act, alpha=alpha)["H"]
    nd, ns = _check_close(q, s, ref)
    assert nd <= q.size // 200 and ns <= s.size // 100


def test_fp8_non_finite_and_zero_k():
    M, K, N = 40, 128, 64
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=3)
    X[0, 5] = float("inf")
    q, s = run(X, Wg, Wu)
    assert np.all(s[0] == 0xFF) and np.all((q[0] & 0x7F) == 0x7F)
    ref = oracle.swiglu_fwd_f64(f64(X[1:]), f64(Wg), f64(Wu))["H"]
    _check_close(q[1:], s[1:], ref)
    # K == 0: h = 0, all codes 0
    Z = torch.empty((M, 0), dtype=torch.bfloat16)
    W0 = torch.empty((N, 0), dtype=torch.bfloat16)
    Hq, Hs = _capi.swiglu_fwd_fp8(*to_dev(Z, W0, W0))
    torch.cuda.synchronize()
    assert not bool(Hq.any()) and not bool(Hs.any())


def test_fp8_full_size_sampled():
    """Prefill size (M=8192, K=4096, N=14336): sampled full rows against the
    oracle's quantisation of the same rows."""
    M, K, N = 8192, 4096, 14336
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, seed=41)
    q, s = run(X, Wg, Wu)
    rows = np.array([0, 1, 127, 128, 4095, 5000, 8190, 8191])
    ref = oracle.swiglu_fwd_f64(f64(X[rows]), f64(Wg), f64(Wu))["H"]
    nd, ns = _check_close(q[rows], s[rows], ref)
    assert nd <= ref.size // 200 and ns <= s[rows].size // 100
