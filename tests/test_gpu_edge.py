"""Non-finite, extreme and subnormal operands on every forward route, element
by element against the fp64 oracle.

The bf16 output is round-to-nearest-even with no saturation and NaN/Inf
propagate as IEEE arithmetic of the definition gives them (the NOSAT,
NaN-preserving casts of "quant: add SwiGLU forward/backward VMI kernels",
implementation notes, whose validation section lists non-finite inputs among
its adversarial cases).  So, per output element:
  * NaN exactly where the oracle's H is NaN;
  * the same signed infinity where the oracle's H is infinite or rounds to
    infinity in the output type (|h| >= the midpoint between the largest
    finite value and 2^128);
  * finite and within the usual tolerance everywhere else.

Cases, each on the decode kernel (M = 1, 8, and the compact-X layout of the
weights-stable launch), the tcgen05 weight stream (M = 16, 128), the dual GEMM
(M = 129, 300) and the fp32 3xTF32 GEMM (M = 4, 129):
  nonfinite_w   NaN and +-Inf planted in rows of Wg and Wu;
  nonfinite_x   NaN, +Inf and -Inf planted in rows of X, one of them above a
                zero weight (Inf * 0 = NaN);
  gates         gate pre-activations in the tails (+-40, +-88.5, +-90, +-104,
                the silu minimum near -1.2785) with random u: one-hot X rows
                make G a chosen weight column exactly;
  overflow      one-hot X rows selecting (g, u) pairs whose product exceeds
                the output's range (+Inf, -Inf), sits exactly on the rounding
                midpoint to infinity (a tie, rounds to infinity), or equals the
                largest finite value (stays finite);
  subnormal     subnormal X times weights near 2^127, and X near 2^127 times
                subnormal weights, so that the products are O(1): an operand
                flushed to zero would change H by O(1)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (FP32_FWD_TOL, assert_guards_intact, assert_ieee_close, dev,
                      guarded_empty, f64)
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu

# (id, M, K, N, dtype, route, weights_stable)
ROUTES = [
    ("decode_m1", 1, 256, 512, "bf16", _capi.ROUTE_DECODE_BF16, False),
    ("decode_m8", 8, 1536, 1032, "bf16", _capi.ROUTE_DECODE_BF16, False),
    ("decode_m3_compact_x", 3, 4096, 264, "bf16", _capi.ROUTE_DECODE_BF16, True),
    ("decode_m8_pdl", 8, 1536, 1032, "bf16", _capi.ROUTE_DECODE_BF16, True),
    ("stream_m16", 16, 256, 520, "bf16", _capi.ROUTE_STREAM_TC_BF16, False),
    ("stream_m128", 128, 512, 264, "bf16", _capi.ROUTE_STREAM_TC_BF16, True),
    ("gemm_m129", 129, 264, 392, "bf16", _capi.ROUTE_GEMM_BF16, False),
    ("gemm_m300", 300, 520, 136, "bf16", _capi.ROUTE_GEMM_BF16, False),
    ("fp32_m4", 4, 132, 136, "f32", _capi.ROUTE_GEMM_TF32X3, False),
    ("fp32_m129", 129, 264, 264, "f32", _capi.ROUTE_GEMM_TF32X3, False),
]

CASES = ["nonfinite_w", "nonfinite_x", "gates", "overflow", "subnormal"]

INF, NAN = np.inf, np.nan


def _base(M, K, N, dtype, seed):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, dtype, seed=seed)
    return (X.float().numpy().copy(), Wg.float().numpy().copy(), Wu.float().numpy().copy())


def _store(a, dtype):
    """Back to the storage dtype; every value planted here is representable."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        b = t.to(torch.bfloat16)
        assert np.array_equal(b.float().numpy(), a, equal_nan=True), "value not representable"
        return b
    return t


def build(case, M, K, N, dtype, seed):
    X, Wg, Wu = _base(M, K, N, dtype, seed)
    if case == "nonfinite_w":
        Wg[N // 3, K // 5] = NAN
        Wg[N // 2, 2] = INF
        Wg[(2 * N) // 3, K - 1] = -INF
        Wu[N - 1, K // 2] = -INF
        Wu[5 % N, 0] = NAN
        Wu[(N // 2 + 7) % N, 3] = INF
    elif case == "nonfinite_x":
        X[0, 1] = INF
        Wg[1, 1] = 0.0                  # Inf * 0 = NaN in G[0, 1]
        Wu[2, 1] = 0.0                  # and in U[0, 2]
        if M >= 2:
            X[M - 1, K - 1] = -INF
        if M >= 3:
            X[M // 2, K // 3] = NAN
    elif case == "gates":
        k0 = 3
        vals = np.array([40.0, -40.0, 90.0, -90.0, -1.2785, 17.0, 0.0, -0.5, 88.5, -88.5,
                         104.0, -104.0, 1.0, -3.0], dtype=np.float32)
        Wg[:, k0] = vals[np.arange(N) % len(vals)]
        r = np.random.Generator(np.random.PCG64(seed + 11))
        Wu[:, k0] = (4.0 * r.standard_normal(N)).astype(np.float32)
        for m in range(0, M, 2):          # one-hot rows: G = Wg[:, k0], U = Wu[:, k0]
            X[m, :] = 0.0
            X[m, k0] = 1.0
        if dtype == "bf16":
            Wg = torch.from_numpy(Wg).to(torch.bfloat16).float().numpy()
            Wu = torch.from_numpy(Wu).to(torch.bfloat16).float().numpy()
    elif case == "overflow":
        p = 2.0
        if dtype == "bf16":
            pairs = [(p ** 70, p ** 70),                       # h = 2^140 -> +Inf
                     (p ** 70, -p ** 70),                      # -> -Inf
                     (73 * p ** 60, 7 * p ** 59),              # h = (2^9-1) 2^119: tie -> +Inf
                     (17 * p ** 60, 15 * p ** 60),             # h = 255 * 2^120: largest finite
                     (17 * p ** 60, -15 * p ** 60),            # -largest finite
                     (-p ** 70, 3.0),                          # silu(-2^70) = -0: h = -0
                     (17 * p ** 64, 0.0),                      # u = 0: h = 0
                     (p ** 64, p ** 63)]                       # h = 2^127: finite
        else:
            pairs = [(p ** 70, p ** 70),
                     (p ** 70, -p ** 70),
                     (18631 * p ** 52, 1801 * p ** 51),        # (2^25-1) 2^103: tie -> +Inf
                     (4095 * p ** 52, 4097 * p ** 52),         # (2^24-1) 2^104: FLT_MAX
                     (4095 * p ** 52, -4097 * p ** 52),
                     (-p ** 70, 3.0),
                     (17 * p ** 64, 0.0),
                     (p ** 64, p ** 63)]
        J = 4
        X[:, :] = 0.0
        for m in range(M):
            X[m, m % J] = 1.0
        for j in range(J):
            for n in range(N):
                g, u = pairs[(n + j) % len(pairs)]
                Wg[n, j] = g
                Wu[n, j] = u
    elif case == "subnormal":
        assert K >= 128
        S1 = np.arange(0, 32)              # subnormal X * large W
        S2 = np.arange(64, 96)             # large X * subnormal W
        r = np.random.Generator(np.random.PCG64(seed + 17))
        c = np.array([1.0, -1.0, 1.5, 0.5, -0.75], dtype=np.float32)
        Wg[:, S1] = (2.0 ** 127) * c[r.integers(0, len(c), (N, 32))]
        Wu[:, S1] = (2.0 ** 127) * c[r.integers(0, len(c), (N, 32))]
        d = np.array([64.0, -64.0, 96.0, 32.0, -96.0], dtype=np.float32)   # x 2^-133
        Wg[:, S2] = (2.0 ** -133) * d[r.integers(0, len(d), (N, 32))]
        Wu[:, S2] = (2.0 ** -133) * d[r.integers(0, len(d), (N, 32))]
        X[:, S1] = 0.0
        X[:, S2] = 0.0
        for m in range(M):
            if m % 3 == 0:
                X[m, :] = 0.0
                X[m, S1] = 2.0 ** -127          # subnormal in bf16 and fp32
            elif m % 3 == 1:
                X[m, :] = 0.0
                X[m, S2] = 2.0 ** 127
    else:
        raise ValueError(case)
    return _store(X, dtype), _store(Wg, dtype), _store(Wu, dtype)


def fp32_bound(ref):
    G, U, H, AG, AU = ref["G"], ref["U"], ref["H"], ref["AG"], ref["AU"]
    with np.errstate(all="ignore"):
        s = 1.0 / (1.0 + np.exp(-np.clip(G, -700, 700)))
        silu = G * s
        dsilu = s * (1.0 + G * (1.0 - s))
        return FP32_FWD_TOL * (np.abs(H) + np.abs(silu) * AU + np.abs(U) * np.abs(dsilu) * AG) \
            + 1e-30


def run(X, Wg, Wu, route, weights_stable, return_gu=False):
    M, K = X.shape
    N = Wg.shape[0]
    Xd, Wgd, Wud = (t.to(dev()) for t in (X, Wg, Wu))
    full, H = guarded_empty(M * N, X.dtype)
    out = _capi.swiglu_fwd(Xd, Wgd, Wud, H.view(M, N), weights_stable=weights_stable,
                           return_gu=return_gu)
    st = _capi.swiglu_sync_status()
    assert st == _capi.SWIGLU_OK, _capi.status_string(st)
    assert _capi.swiglu_last_route() == route
    assert_guards_intact(full)
    if return_gu:
        return tuple(t.cpu() for t in out)
    return H.view(M, N).cpu()


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("rid,M,K,N,dtype,route,ws", ROUTES, ids=[r[0] for r in ROUTES])
def test_forward_edge(rid, M, K, N, dtype, route, ws, case):
    assert _capi.swiglu_route_for(M, K, N, 0 if dtype == "bf16" else 1) == route
    X, Wg, Wu = build(case, M, K, N, dtype, seed=M * 31 + K)
    H = run(X, Wg, Wu, route, ws)
    ref = oracle.swiglu_fwd(X, Wg, Wu, dtype, want_magnitudes=(dtype == "f32"))
    counts = assert_ieee_close(f64(H), ref["H"], f"{rid} {case}", dtype,
                               fp32_bound(ref) if dtype == "f32" else None)
    # the planted values really reach the output classes they are meant to
    if case.startswith("nonfinite"):
        assert counts["nan"] > 0
        assert counts["finite"] > 0 or (case == "nonfinite_x" and M <= 3)  # every row planted
    if case == "overflow":
        assert counts["inf"] > 0 and counts["finite"] > 0
        assert np.any(np.abs(f64(H)) == (255 * 2.0 ** 120 if dtype == "bf16"
                                         else float(np.finfo(np.float32).max)))


@pytest.mark.parametrize("case", ["nonfinite_w", "nonfinite_x", "overflow"])
@pytest.mark.parametrize("rid,M,K,N,dtype,route,ws",
                         [r for r in ROUTES if r[4] == "bf16"], ids=[r[0] for r in ROUTES
                                                                     if r[4] == "bf16"])
def test_training_forward_edge(rid, M, K, N, dtype, route, ws, case):
    """The training forward's stored G and U (each the fp32 accumulator
    rounded once) follow the same rules as H."""
    X, Wg, Wu = build(case, M, K, N, dtype, seed=M * 37 + K)
    H, G, U = run(X, Wg, Wu, route, ws, return_gu=True)
    ref = oracle.swiglu_fwd(X, Wg, Wu, dtype)
    assert_ieee_close(f64(H), ref["H"], f"{rid} {case} H")
    assert_ieee_close(f64(G), ref["G"], f"{rid} {case} G")
    assert_ieee_close(f64(U), ref["U"], f"{rid} {case} U")


@pytest.mark.parametrize("combined", [False, True], ids=["separate", "one_launch"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_backward_gemms_nonfinite(dtype, combined):
    """dX = dG Wg + dU Wu, dWg = dG^T X, dWu = dU^T X with NaN and +-Inf planted
    in dG, dU, Wg, Wu and X (and zeros under some of them, Inf * 0 = NaN):
    the same classes as the oracle's IEEE double sums, finite outputs within
    the usual tolerance (fp32: 1e-5 of the sum of the terms' magnitudes)."""
    M, K, N = 130, 136, 264
    X, Wg, Wu = _base(M, K, N, dtype, seed=5)
    dG = synth.normal((M, N), 41, dtype=dtype).float().numpy().copy()
    dU = synth.normal((M, N), 42, dtype=dtype).float().numpy().copy()
    dG[3, 5] = INF
    Wg[5, 7] = 0.0                      # dX[3, 7] gets Inf * 0
    dU[7, 9] = NAN
    Wg[11, 2] = -INF
    Wu[20, 40] = INF
    X[4, 6] = INF
    dG[4, 100] = 0.0                    # dWg[100, 6] gets 0 * Inf
    X[9, 30] = -INF
    dGt, dUt, Xt, Wgt, Wut = (_store(a, dtype) for a in (dG, dU, X, Wg, Wu))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    dGd, dUd, Xd, Wgd, Wud = (t.to(dev()) for t in (dGt, dUt, Xt, Wgt, Wut))
    if combined:
        dX, dWg, dWu = _capi.swiglu_bwd_gemms(dGd, dUd, Wgd, Wud, Xd)
    else:
        dX = _capi.swiglu_bwd_dx(dGd, dUd, Wgd, Wud)
        dWg, dWu = _capi.swiglu_bwd_dw(dGd, dUd, Xd)
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert dX.dtype == tdt
    o64 = [a.astype(np.float64) for a in (dG, dU, Wg, Wu, X)]
    rX = oracle.bwd_dx_f64(o64[0], o64[1], o64[2], o64[3])
    rWg, rWu = oracle.bwd_dw_f64(o64[0], o64[1], o64[4])

    def fin(a):
        return np.where(np.isfinite(a), np.abs(a), 0.0)

    bX = 1e-5 * (fin(o64[0]) @ fin(o64[2]) + fin(o64[1]) @ fin(o64[3])) + 1e-30
    bWg = 1e-5 * (fin(o64[0]).T @ fin(o64[4])) + 1e-30
    bWu = 1e-5 * (fin(o64[1]).T @ fin(o64[4])) + 1e-30
    c1 = assert_ieee_close(f64(dX), rX, f"dX {dtype}", dtype, bX)
    c2 = assert_ieee_close(f64(dWg), rWg, f"dWg {dtype}", dtype, bWg)
    c3 = assert_ieee_close(f64(dWu), rWu, f"dWu {dtype}", dtype, bWu)
    for c in (c1, c2, c3):
        assert c["nan"] > 0 and c["inf"] > 0 and c["finite"] > 0
