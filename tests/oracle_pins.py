"""Pins for the fp64 oracle: checks against facts fixed by the mathematics,
by an independent library routine, or by brute force -- never against the
oracle's own formula retyped.

Every pin takes an ``oracle.Oracle`` instance and raises AssertionError on a
mismatch, so the same suite runs against the committed oracle and against
copies with a mistake planted in them (test_oracle_mutants.py), which shows
that each plausible mistake trips at least one pin.

What pins what:
  scalar_closed_forms   sigmoid/silu/silu' at points with known values, the
                        identities silu(-x) = silu(x) - x and
                        sigmoid(x) + sigmoid(-x) = 1, the silu minimum at
                        x* = -1 - W(1/e) with value -W(1/e) (W = Lambert W,
                        computed here by Newton's method), the limits
                        silu(x) -> x and silu(x) -> 0, and silu' against a
                        central difference of silu.
  fwd_library           G, U against numpy float64 matmul (independent BLAS);
                        the magnitudes AG, AU against |X| @ |W|^T.
  fwd_brute_force       G, U against exactly rounded sums (math.fsum) of the
                        exact products, on tiny shapes.
  fwd_gate_up_roles     H(Wg) - H(-Wg) = G * U elementwise (from the identity
                        above), with G, U from numpy: fixes which operand is
                        the gate and the sign convention.
  fwd_zero_cases        U = 0 => H = 0, Wg = 0 => H = 0.
  fwd_linear_in_up      H(a Wu) = a H.
  fwd_one_hot           X = e_k selects weight column k: G = Wg[:, k] and
                        U = Wu[:, k] exactly.
  fwd_asymptotes        G = +40 => H ~ 40 U, G = -40 => H ~ 0.
  fwd_points            the sampled forward equals the full forward.
  fwd_nonfinite         NaN and +-Inf in X, Wg, Wu: silu(+Inf) = +Inf,
                        silu(-Inf) and silu(NaN) are NaN as torch's silu gives
                        them in float64 (an independent library routine); G, U
                        against a brute-force loop of Python float products;
                        H against torch's silu(G) * U, class by class (NaN,
                        +-Inf, finite) and value by value.
  bf16_decoder          all 65536 bf16 patterns decode like torch's bf16.
  dswiglu_finite_diff   dG, dU against central differences of the forward.
  dswiglu_special       dh = 0, u = 0, g = 0, g = +-40, g = x*.
  dswiglu_storage       the bf16 and fp32 entry points agree with the double
                        one on the decoded values.
  gelu_closed_forms     GELU(tanh): value and slope at 0, the identity
                        gelu(x) - gelu(-x) = x, the limits, torch's
                        gelu(approximate="tanh") in float64 (an independent
                        library routine), and gelu' against central differences.
  variants_fwd          act(alpha g) u: G, U do not depend on the variant;
                        H(Wg) - H(-Wg) = G U for GELU too (from its identity);
                        H(alpha, Wg) = H(1, alpha Wg) for alpha a power of two
                        (the multiplier acts on the gate pre-activation).
  variants_bwd          dG, dU of the variants against central differences of
                        the variant forward, and dU = dh act(alpha g).
  gelu_high_precision   gelu, gelu' against the tanh definition in 120-digit
                        mpmath arithmetic, x in [-12, 8].
  e4m3_codec            the e4m3 decode of all 256 codes and the round-to-
                        nearest-even encode of ties, subnormals and random
                        values against torch's float8_e4m3fn conversion.
  ue8m0_scale           closed forms of the block exponent (powers of two
                        times 448, just above them, clamps).
  quant_blocks          per-(1,32)-block quantisation: dequantised values
                        within half an e4m3 step, the block maximum lands in
                        (224, 448], ragged last block, non-finite blocks.
  backward_gemms        dX, dWg, dWu against numpy matmul, and the whole chain
                        (forward, dSwiGLU, backward GEMMs) against central
                        differences of the scalar loss sum(dH * H) in X, Wg, Wu.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def lambert_w_inv_e() -> float:
    """W(1/e): the root of w e^w = 1/e, by Newton's method from w = 0.3."""
    w = 0.3
    target = math.exp(-1.0)
    for _ in range(60):
        f = w * math.exp(w) - target
        w -= f / (math.exp(w) * (1.0 + w))
    return w


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


def _bf16_exact(a: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 and back (torch RNE), so that every
    product of two such values is exact in double."""
    return torch.from_numpy(a).to(torch.bfloat16).to(torch.float64).numpy()


# ---- scalar definitions ---------------------------------------------------

def scalar_closed_forms(o):
    assert o.silu(0.0) == 0.0
    assert o.sigmoid(0.0) == 0.5
    assert o.dsilu(0.0) == 0.5
    # sigmoid(ln 3) = 1 / (1 + 1/3) = 3/4 and sigmoid(-ln 3) = 1/4.
    assert abs(o.sigmoid(math.log(3.0)) - 0.75) < 1e-15
    assert abs(o.sigmoid(-math.log(3.0)) - 0.25) < 1e-15
    # Limits: silu(30) = 30 / (1 + e^-30) is 30 - 2.8e-12; silu(-40) ~ -1.7e-16.
    s30 = o.silu(30.0)
    assert 0.0 < 30.0 - s30 < 1e-11, s30
    assert abs(o.silu(-40.0)) < 1e-15
    assert o.silu(-40.0) < 0.0
    for x in np.linspace(-25.0, 25.0, 101):
        x = float(x)
        # silu(-x) = -x (1 - sigmoid(x)) = silu(x) - x
        assert abs(o.silu(-x) - (o.silu(x) - x)) <= 1e-14 * max(1.0, abs(x)), x
        assert abs(o.sigmoid(x) + o.sigmoid(-x) - 1.0) <= 4.5e-16, x
        # silu' against a central difference of silu (step 1e-5: truncation
        # ~1e-11, rounding ~1e-11).
        h = 1e-5
        fd = (o.silu(x + h) - o.silu(x - h)) / (2.0 * h)
        assert abs(o.dsilu(x) - fd) < 1e-8, (x, o.dsilu(x), fd)
    # Minimum of silu: silu'(x) = 0 <=> x = -(1 + e^x) <=> x* = -1 - W(1/e),
    # where silu(x*) = x* + 1 = -W(1/e).
    w = lambert_w_inv_e()
    xs = -1.0 - w
    assert abs(o.silu(xs) - (-w)) < 1e-15, (o.silu(xs), -w)
    assert abs(o.dsilu(xs)) < 1e-15, o.dsilu(xs)
    assert o.silu(xs - 1e-3) > o.silu(xs) and o.silu(xs + 1e-3) > o.silu(xs)


# ---- forward --------------------------------------------------------------

def _random_problem(M, K, N, seed, scale_w=None):
    r = _rng(seed)
    sw = (1.0 / math.sqrt(K)) if scale_w is None else scale_w
    X = _bf16_exact(r.standard_normal((M, K)))
    Wg = _bf16_exact(r.standard_normal((N, K)) * sw)
    Wu = _bf16_exact(r.standard_normal((N, K)) * sw)
    return X, Wg, Wu


def fwd_library(o):
    for (M, K, N, seed) in [(4, 256, 512, 0), (3, 40, 24, 1), (8, 1536, 64, 2),
                            (130, 72, 136, 3)]:
        X, Wg, Wu = _random_problem(M, K, N, seed)
        out = o.swiglu_fwd_f64(X, Wg, Wu, want_magnitudes=True)
        G_ref = X @ Wg.T
        U_ref = X @ Wu.T
        bound_g = 1e-13 * (np.abs(X) @ np.abs(Wg).T) + 1e-300
        bound_u = 1e-13 * (np.abs(X) @ np.abs(Wu).T) + 1e-300
        assert np.all(np.abs(out["G"] - G_ref) <= bound_g), (M, K, N)
        assert np.all(np.abs(out["U"] - U_ref) <= bound_u), (M, K, N)
        assert np.allclose(out["AG"], np.abs(X) @ np.abs(Wg).T, rtol=1e-13, atol=0)
        assert np.allclose(out["AU"], np.abs(X) @ np.abs(Wu).T, rtol=1e-13, atol=0)


def fwd_brute_force(o):
    for (M, K, N, seed) in [(2, 7, 3, 10), (3, 16, 5, 11), (1, 33, 2, 12)]:
        X, Wg, Wu = _random_problem(M, K, N, seed)
        out = o.swiglu_fwd_f64(X, Wg, Wu, want_magnitudes=True)
        for m in range(M):
            for n in range(N):
                # products of bf16 values are exact in double; fsum rounds once
                g = math.fsum(float(X[m, k]) * float(Wg[n, k]) for k in range(K))
                u = math.fsum(float(X[m, k]) * float(Wu[n, k]) for k in range(K))
                tol_g = K * 2.0 ** -53 * out["AG"][m, n]
                tol_u = K * 2.0 ** -53 * out["AU"][m, n]
                assert abs(out["G"][m, n] - g) <= tol_g, (m, n)
                assert abs(out["U"][m, n] - u) <= tol_u, (m, n)


def fwd_gate_up_roles(o):
    X, Wg, Wu = _random_problem(5, 64, 48, 20, scale_w=0.3)
    H_pos = o.swiglu_fwd_f64(X, Wg, Wu)["H"]
    H_neg = o.swiglu_fwd_f64(X, -Wg, Wu)["H"]
    GU = (X @ Wg.T) * (X @ Wu.T)
    scale = np.abs(X) @ np.abs(Wg).T * np.abs(X @ Wu.T) + 1e-300
    assert np.all(np.abs((H_pos - H_neg) - GU) <= 1e-12 * scale)
    # and the gate really is nonlinear: H is not G*U/2 everywhere
    assert np.max(np.abs(H_pos - 0.5 * GU)) > 1e-3


def fwd_zero_cases(o):
    X, Wg, Wu = _random_problem(4, 32, 16, 30)
    assert np.all(o.swiglu_fwd_f64(X, Wg, np.zeros_like(Wu))["H"] == 0.0)
    assert np.all(o.swiglu_fwd_f64(X, np.zeros_like(Wg), Wu)["H"] == 0.0)
    # K = 0: empty sums
    e = o.swiglu_fwd_f64(np.zeros((3, 0)), np.zeros((2, 0)), np.zeros((2, 0)))
    assert np.all(e["G"] == 0.0) and np.all(e["H"] == 0.0)


def fwd_linear_in_up(o):
    X, Wg, Wu = _random_problem(4, 64, 32, 40)
    H = o.swiglu_fwd_f64(X, Wg, Wu)["H"]
    assert np.array_equal(o.swiglu_fwd_f64(X, Wg, 2.0 * Wu)["H"], 2.0 * H)
    H3 = o.swiglu_fwd_f64(X, Wg, -3.0 * Wu)["H"]
    assert np.allclose(H3, -3.0 * H, rtol=1e-14, atol=1e-300)


def fwd_one_hot(o):
    r = _rng(50)
    K, N = 24, 40
    _, Wg, Wu = _random_problem(1, K, N, 51, scale_w=1.0)
    ks = [0, 5, K - 1, 13]
    X = np.zeros((len(ks), K))
    for m, k in enumerate(ks):
        X[m, k] = 1.0
    out = o.swiglu_fwd_f64(X, Wg, Wu)
    for m, k in enumerate(ks):
        assert np.array_equal(out["G"][m], Wg[:, k]), (m, k)
        assert np.array_equal(out["U"][m], Wu[:, k]), (m, k)
        for n in range(N):
            assert out["H"][m, n] == o.silu(Wg[n, k]) * Wu[n, k]
    del r


def fwd_asymptotes(o):
    # X = [1, 0...], Wg[:,0] = +-40 => G = +-40 exactly; U = Wu[:,0].
    N, K = 16, 8
    X = np.zeros((1, K))
    X[0, 0] = 1.0
    r = _rng(60)
    Wu = _bf16_exact(r.standard_normal((N, K)))
    for gval in (40.0, -40.0):
        Wg = np.zeros((N, K))
        Wg[:, 0] = gval
        H = o.swiglu_fwd_f64(X, Wg, Wu)["H"][0]
        U = Wu[:, 0]
        if gval > 0:
            assert np.allclose(H, 40.0 * U, rtol=1e-15, atol=0)
        else:
            assert np.all(np.abs(H) <= 40.0 * math.exp(-40.0) * np.abs(U) * 1.01)


def fwd_points(o):
    from up_projection_b200 import synth  # seeded inputs only
    M, K, N = 9, 136, 72
    for dtype in ("bf16", "f32"):
        X, Wg, Wu = synth.swiglu_inputs(M, K, N, dtype=dtype, seed=7)
        full = o.swiglu_fwd(X, Wg, Wu, dtype=dtype, want_magnitudes=True)
        r = _rng(70)
        im = r.integers(0, M, size=200)
        inn = r.integers(0, N, size=200)
        pts = o.swiglu_fwd_points(X, Wg, Wu, im, inn, dtype=dtype)
        for key in ("G", "U", "H", "AG", "AU"):
            assert np.array_equal(pts[key], full[key][im, inn]), (dtype, key)
        # and against numpy on the decoded operands
        Xd = X.to(torch.float64).numpy()
        Wgd = Wg.to(torch.float64).numpy()
        G_np = np.einsum("ik,ik->i", Xd[im], Wgd[inn])
        assert np.all(np.abs(pts["G"] - G_np) <= 1e-13 * pts["AG"] + 1e-300)


def _same_ieee(a, b, rtol=0.0):
    """a and b agree element by element: NaN where the other is NaN, the same
    signed infinity, and finite values within rtol (relative)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    na, nb = np.isnan(a), np.isnan(b)
    if not np.array_equal(na, nb):
        return False
    ia, ib = np.isinf(a), np.isinf(b)
    if not np.array_equal(ia, ib) or not np.array_equal(a[ia], b[ib]):
        return False
    f = ~(na | ia)
    return bool(np.all(np.abs(a[f] - b[f]) <= rtol * np.abs(b[f])))


def fwd_nonfinite(o):
    inf, nan = math.inf, math.nan
    # closed forms, and torch's float64 silu at the same points
    assert o.silu(inf) == inf and math.isnan(o.silu(-inf)) and math.isnan(o.silu(nan))
    pts = torch.tensor([inf, -inf, nan, -90.0, 0.0, 90.0], dtype=torch.float64)
    theirs = torch.nn.functional.silu(pts).numpy()
    ours = np.array([o.silu(float(v)) for v in pts])
    assert _same_ieee(ours, theirs, rtol=1e-15)
    # a small problem with non-finite operands planted in rows of each input
    M, K, N = 5, 9, 7
    X, Wg, Wu = _random_problem(M, K, N, 90)
    X[1, 2] = nan
    X[2, 4] = inf
    X[3, 0] = -inf
    Wg[2, 5] = nan
    Wg[4, 1] = inf
    Wu[5, 7] = -inf
    Wu[6, 3] = nan
    Wg[0, 4] = 0.0          # X[2, 4] * Wg[0, 4] = Inf * 0 = NaN
    out = o.swiglu_fwd_f64(X, Wg, Wu)
    G = np.empty((M, N))
    U = np.empty((M, N))
    for m in range(M):
        for n in range(N):
            g = 0.0
            u = 0.0
            for k in range(K):
                g += float(X[m, k]) * float(Wg[n, k])
                u += float(X[m, k]) * float(Wu[n, k])
            G[m, n] = g
            U[m, n] = u
    assert _same_ieee(out["G"], G, rtol=1e-13) and _same_ieee(out["U"], U, rtol=1e-13)
    H = (torch.nn.functional.silu(torch.from_numpy(G)) * torch.from_numpy(U)).numpy()
    assert _same_ieee(out["H"], H, rtol=1e-13)
    # every class occurs, so the comparison above is not vacuous
    assert np.isnan(out["H"]).any() and np.isposinf(out["H"]).any()
    assert np.isneginf(out["H"]).any() and np.isfinite(out["H"]).any()
    assert np.isnan(out["H"][1]).all() and np.isnan(out["H"][:, 2]).all()


def bf16_decoder(o):
    bits = np.arange(65536, dtype=np.uint16)
    ours = o.decode_bf16(bits)
    theirs = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16) \
        .to(torch.float64).numpy()
    nan = np.isnan(theirs)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], theirs[~nan])
    # signed zeros keep their sign
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(theirs[~nan]))


# ---- backward ------------------------------------------------------------

def _fwd_scalar(o, g, u):
    """h(g, u) = silu(g) u through the oracle's FORWARD path (K = 1)."""
    return float(o.swiglu_fwd_f64(np.array([[1.0]]), np.array([[g]]),
                                  np.array([[u]]))["H"][0, 0])


def dswiglu_finite_diff(o):
    r = _rng(80)
    g = np.concatenate([r.standard_normal(40) * 3.0, [0.0, -1.2784, 5.0, -6.0]])
    u = r.standard_normal(g.size)
    dh = r.standard_normal(g.size)
    dG, dU = o.dswiglu_f64(dh, g, u)
    d = 1e-6
    for i in range(g.size):
        fd_g = (_fwd_scalar(o, g[i] + d, u[i]) - _fwd_scalar(o, g[i] - d, u[i])) / (2 * d)
        fd_u = (_fwd_scalar(o, g[i], u[i] + d) - _fwd_scalar(o, g[i], u[i] - d)) / (2 * d)
        sg = abs(dh[i]) * (abs(u[i]) + 1.0)
        su = abs(dh[i]) * (abs(g[i]) + 1.0)
        assert abs(dG[i] - dh[i] * fd_g) <= 2e-8 * sg, (i, g[i], dG[i], dh[i] * fd_g)
        assert abs(dU[i] - dh[i] * fd_u) <= 2e-8 * su, (i, g[i], dU[i], dh[i] * fd_u)


def dswiglu_special(o):
    w = lambert_w_inv_e()
    g = np.array([0.0, 1.0, 40.0, -40.0, -1.0 - w, 2.0])
    u = np.array([3.0, 0.0, 2.0, 2.0, 1.5, -1.0])
    dh = np.array([2.0, 1.0, 1.0, 1.0, 1.0, 0.0])
    dG, dU = o.dswiglu_f64(dh, g, u)
    assert dU[0] == 0.0 and dG[0] == 2.0 * 3.0 * 0.5      # g = 0
    assert dG[1] == 0.0                                    # u = 0
    assert abs(dU[1] - o.silu(1.0)) < 1e-16
    assert abs(dU[2] - 40.0) < 1e-14 and abs(dG[2] - 2.0) < 1e-14   # g -> +inf
    assert abs(dU[3]) < 1e-15 and abs(dG[3]) < 1e-15                # g -> -inf
    assert abs(dG[4]) < 1e-15                               # silu'(x*) = 0
    assert abs(dU[4] - 1.0 * (-w)) < 1e-15                  # silu(x*) = -W(1/e)
    assert dG[5] == 0.0 and dU[5] == 0.0                   # dh = 0


def dswiglu_storage(o):
    from up_projection_b200 import synth
    for dtype in ("bf16", "f32"):
        dH, G, U = synth.dswiglu_inputs(1000, dtype=dtype, seed=9)
        dG, dU = o.dswiglu(dH, G, U, dtype=dtype)
        dG2, dU2 = o.dswiglu_f64(o.decode(dH, dtype), o.decode(G, dtype),
                                 o.decode(U, dtype))
        assert np.array_equal(dG, dG2) and np.array_equal(dU, dU2), dtype


def gelu_closed_forms(o):
    assert o.gelu_tanh(0.0) == 0.0
    assert o.dgelu_tanh(0.0) == 0.5
    assert o.act(1.3, 1) == o.gelu_tanh(1.3) and o.act(1.3, 0) == o.silu(1.3)
    assert abs(o.gelu_tanh(10.0) - 10.0) < 1e-15
    assert abs(o.gelu_tanh(-10.0)) < 1e-15
    xs = np.linspace(-8.0, 8.0, 161)
    ref = torch.nn.functional.gelu(torch.from_numpy(xs), approximate="tanh").numpy()
    for x, r in zip(xs, ref):
        x = float(x)
        assert abs(o.gelu_tanh(x) - r) <= 1e-15 * max(1.0, abs(x)), (x, o.gelu_tanh(x), r)
        # gelu(x) - gelu(-x) = x  (the tanh factor is odd)
        assert abs(o.gelu_tanh(x) - o.gelu_tanh(-x) - x) <= 1e-14 * max(1.0, abs(x)), x
        h = 1e-5
        fd = (o.gelu_tanh(x + h) - o.gelu_tanh(x - h)) / (2.0 * h)
        assert abs(o.dgelu_tanh(x) - fd) < 1e-8, (x, o.dgelu_tanh(x), fd)
        assert o.dact(x, 1) == o.dgelu_tanh(x) and o.dact(x, 0) == o.dsilu(x)


def gelu_high_precision(o):
    """gelu and gelu' against the definition x/2 (1 + tanh(c(x + a x^3)))
    evaluated in 120-digit arithmetic (mpmath), where 1 + tanh(y) does not
    cancel: relative agreement over the whole range, including x < -5 where
    a double-precision tanh form loses its digits."""
    import mpmath
    mpmath.mp.dps = 120
    c = mpmath.sqrt(2 / mpmath.pi)
    a = mpmath.mpf("0.044715")

    def g(x):
        return x / 2 * (1 + mpmath.tanh(c * (x + a * x ** 3)))
    for xf in list(np.linspace(-12.0, 8.0, 81)) + [-6.578, -7.3, -9.5, 1e-3, -1e-3]:
        x = mpmath.mpf(float(xf))
        ref = g(x)
        dref = mpmath.diff(g, x)
        v, dv = o.gelu_tanh(float(xf)), o.dgelu_tanh(float(xf))
        # e^(2y) turns the rounding of its double argument (a few ulp of
        # |2y|) into a relative error of about |2y| ulp: the bound scales
        # with |2y| (about 10 ulp at x = 0, 2.6e-13 at x = -12).
        z = abs(2 * float(c) * (float(xf) + 0.044715 * float(xf) ** 3))
        tol = 2.2e-16 * (20.0 + 8.0 * z)
        assert abs(mpmath.mpf(v) - ref) <= tol * abs(ref), (xf, v, ref)
        # gelu' = s + 2 x s (1 - s) y' cancels near the minimum of gelu
        # (x ~ -0.75): relative to the size of its two terms there.
        xv = float(xf)
        sd = float(1 / (1 + mpmath.exp(-2 * c * (x + a * x ** 3))))
        terms = abs(sd) + abs(2 * xv * sd * (1 - sd) * float(c) * (1 + 3 * 0.044715 * xv * xv))
        assert abs(mpmath.mpf(dv) - dref) <= 2 * tol * max(abs(float(dref)), terms) + 1e-300, \
            (xf, dv, dref)
    assert o.gelu_tanh(-10.0) < 0.0 and o.dgelu_tanh(-10.0) != 0.0


def variants_fwd(o):
    X, Wg, Wu = _random_problem(5, 64, 40, 90, scale_w=0.4)
    base = o.swiglu_fwd_f64(X, Wg, Wu)
    GU = (X @ Wg.T) * (X @ Wu.T)
    scale = np.abs(X) @ np.abs(Wg).T * np.abs(X @ Wu.T) + 1e-300
    for act in (0, 1):
        v = o.swiglu_fwd_f64(X, Wg, Wu, act=act, alpha=1.0)
        assert np.array_equal(v["G"], base["G"]) and np.array_equal(v["U"], base["U"])
        if act == 0:
            assert np.array_equal(v["H"], base["H"])
        # act(g) - act(-g) = g for both activations
        vn = o.swiglu_fwd_f64(X, -Wg, Wu, act=act)
        assert np.all(np.abs((v["H"] - vn["H"]) - GU) <= 1e-12 * scale), act
        for alpha in (2.0, 0.5, -4.0):
            a = o.swiglu_fwd_f64(X, Wg, Wu, act=act, alpha=alpha)
            b = o.swiglu_fwd_f64(X, alpha * Wg, Wu, act=act)
            assert np.array_equal(a["H"], b["H"]), (act, alpha)
            assert np.array_equal(a["G"], v["G"])   # G is stored before the multiplier
    # a multiplier really changes H (it is not applied after the activation)
    a = o.swiglu_fwd_f64(X, Wg, Wu, alpha=2.0)["H"]
    assert np.max(np.abs(a - 2.0 * base["H"])) > 1e-3


def variants_bwd(o):
    r = _rng(95)
    g = r.standard_normal(30) * 2.0
    u = r.standard_normal(30)
    dh = r.standard_normal(30)
    d = 1e-6
    for act in (0, 1):
        for alpha in (1.0, 1.7, -0.6):
            dG, dU = o.dswiglu_f64(dh, g, u, act=act, alpha=alpha)

            def h(gg, uu):
                return float(o.swiglu_fwd_f64(np.array([[1.0]]), np.array([[gg]]),
                                              np.array([[uu]]), act=act, alpha=alpha)["H"][0, 0])
            for i in range(g.size):
                fdg = (h(g[i] + d, u[i]) - h(g[i] - d, u[i])) / (2 * d)
                fdu = (h(g[i], u[i] + d) - h(g[i], u[i] - d)) / (2 * d)
                sg = abs(dh[i]) * (abs(u[i]) + 1.0) * (abs(alpha) + 1.0)
                assert abs(dG[i] - dh[i] * fdg) <= 3e-8 * sg, (act, alpha, i)
                assert abs(dU[i] - dh[i] * fdu) <= 3e-8 * abs(dh[i]) * (abs(g[i] * alpha) + 1.0)
                assert dU[i] == dh[i] * o.act(alpha * g[i], act)


def backward_gemms(o):
    r = _rng(120)
    M, K, N = 5, 12, 9
    X = r.standard_normal((M, K))
    Wg = r.standard_normal((N, K)) * 0.4
    Wu = r.standard_normal((N, K)) * 0.4
    dH = r.standard_normal((M, N))
    f = o.swiglu_fwd_f64(X, Wg, Wu)
    dG, dU = o.dswiglu_f64(dH, f["G"], f["U"])
    dX = o.bwd_dx_f64(dG, dU, Wg, Wu)
    dWg, dWu = o.bwd_dw_f64(dG, dU, X)
    assert np.allclose(dX, dG @ Wg + dU @ Wu, rtol=1e-12, atol=1e-14)
    assert np.allclose(dWg, dG.T @ X, rtol=1e-12, atol=1e-14)
    assert np.allclose(dWu, dU.T @ X, rtol=1e-12, atol=1e-14)

    def loss(X_, Wg_, Wu_):
        return float(np.sum(dH * o.swiglu_fwd_f64(X_, Wg_, Wu_)["H"]))
    d = 1e-6
    for (arr, grad, name) in ((X, dX, "X"), (Wg, dWg, "Wg"), (Wu, dWu, "Wu")):
        for idx in [(0, 0), (arr.shape[0] - 1, arr.shape[1] - 1), (2, 5), (1, 7)]:
            p, q = arr.copy(), arr.copy()
            p[idx] += d
            q[idx] -= d
            args_p = [X, Wg, Wu]
            args_q = [X, Wg, Wu]
            i = {"X": 0, "Wg": 1, "Wu": 2}[name]
            args_p[i], args_q[i] = p, q
            fd = (loss(*args_p) - loss(*args_q)) / (2 * d)
            assert abs(fd - grad[idx]) <= 1e-7 * (1 + abs(fd)), (name, idx, fd, grad[idx])


def e4m3_codec(o):
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = o.e4m3_decode(c)
        if np.isnan(ref[c]):
            assert np.isnan(v), c
        else:
            assert v == ref[c] and (np.signbit(v) == np.signbit(ref[c])), (c, v, ref[c])
    finite = np.sort(np.unique(np.abs(ref[np.isfinite(ref)])))
    mids = (finite[:-1] + finite[1:]) / 2           # exact ties between codes
    r = _rng(31)
    vals = np.concatenate([finite, mids, -mids, r.uniform(-448, 448, 3000),
                           r.uniform(-2 ** -6, 2 ** -6, 500), [0.0, -0.0, 2 ** -10, 2 ** -9 * 0.5]])
    t = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, c in zip(vals, t):
        assert o.e4m3_encode(float(v)) == int(c), (v, o.e4m3_encode(float(v)), int(c))
    assert o.e4m3_encode(448.5) == 0x7F and o.e4m3_encode(float("nan")) == 0x7F


def ue8m0_scale(o):
    for k in range(-120, 120, 7):
        a = 448.0 * 2.0 ** k
        assert o.ue8m0_exponent(a) == k
        assert o.ue8m0_exponent(a * (1 + 2 ** -40)) == k + 1
        assert o.ue8m0_exponent(a * (1 - 2 ** -40)) == k
    assert o.ue8m0_exponent(1.0) == -8          # 448 / 256 = 1.75 >= 1 > 0.875
    assert o.ue8m0_exponent(0.0) == -127
    assert o.ue8m0_exponent(1e-300) == -127     # clamped below
    assert o.ue8m0_exponent(1e300) == 127       # clamped above


def quant_blocks(o):
    r = _rng(32)
    H = r.standard_normal((6, 100)) * np.exp(r.uniform(-8, 8, (6, 1)))
    H[2, 40:50] *= 1e3          # one block with a much larger maximum
    H[3, 64:96] = 0.0           # an all-zero block
    q, s = o.quant_e4m3(H)
    assert q.shape == (6, 100) and s.shape == (6, 4)   # ragged last block of 4
    dec = np.vectorize(o.e4m3_decode)
    for m in range(6):
        for b in range(4):
            lo, hi = 32 * b, min(32 * b + 32, 100)
            e = int(s[m, b]) - 127
            blk = H[m, lo:hi]
            d = dec(q[m, lo:hi]) * 2.0 ** e
            if not np.any(blk):
                assert e == -127 and not np.any(d)
                continue
            # the largest element lands in (224, 448] after scaling
            assert 224.0 < np.max(np.abs(blk)) * 2.0 ** -e <= 448.0
            # within half a step of the e4m3 grid (relative 2^-4 for normals,
            # absolute 2^-10 * 2^e in the subnormal range)
            step = np.maximum(np.abs(blk) * 2.0 ** -3, 2.0 ** (e - 9))
            assert np.all(np.abs(d - blk) <= 0.5 * step + 1e-300), (m, b)
    bad = np.zeros((1, 64))
    bad[0, 3] = np.inf
    bad[0, 40] = np.nan
    q, s = o.quant_e4m3(bad)
    assert list(s[0]) == [0xFF, 0xFF] and np.all(q == 0x7F)


ALL_PINS = [scalar_closed_forms, fwd_library, fwd_brute_force,
            fwd_gate_up_roles, fwd_zero_cases, fwd_linear_in_up, fwd_one_hot,
            fwd_asymptotes, fwd_points, fwd_nonfinite, bf16_decoder, dswiglu_finite_diff,
            dswiglu_special, dswiglu_storage, gelu_closed_forms, variants_fwd,
            variants_bwd, backward_gemms, gelu_high_precision, e4m3_codec, ue8m0_scale,
            quant_blocks]
