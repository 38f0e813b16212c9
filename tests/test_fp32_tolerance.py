"""The fp32-mode tolerance is discriminating (CPU only).

Liger-Kernel issue #1383 reports that plain TF32 tensor-core matmuls break
fp32 parity.  Emulating the two arithmetics on the host (operands rounded to
TF32 as the tensor cores see them, products and sums in fp64) shows that the
bound the GPU tests use rejects plain TF32 and accepts the 3xTF32 split
(hi*hi + hi*lo + lo*hi), so passing it is evidence of the split working."""
import numpy as np

import oracle
from up_projection_b200 import synth

TOL = 1e-5


def tf32_rna(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to TF32 (10 explicit mantissa bits), to nearest,
    ties away from zero -- the cvt.rna.tf32.f32 rule."""
    b = a.astype(np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x1000) & 0xFFFFE000
    return b.astype(np.uint32).view(np.float32)


def bound(ref):
    G, U, H = ref["G"], ref["U"], ref["H"]
    s = 1 / (1 + np.exp(-G))
    return TOL * (np.abs(H) + np.abs(G * s) * ref["AU"]
                  + np.abs(U) * np.abs(s * (1 + G * (1 - s))) * ref["AG"])


def silu_mul(G, U):
    return G / (1 + np.exp(-G)) * U


def test_plain_tf32_fails_and_3xtf32_passes():
    M, K, N = 16, 2048, 256
    X, Wg, Wu = (t.numpy() for t in synth.swiglu_inputs(M, K, N, "f32", seed=5))
    ref = oracle.swiglu_fwd(X, Wg, Wu, "f32", want_magnitudes=True)
    b = bound(ref)

    def split(a):
        hi = tf32_rna(a)
        lo = tf32_rna((a - hi).astype(np.float32))
        return hi.astype(np.float64), lo.astype(np.float64)

    # plain TF32: one product of rounded operands
    Gt = tf32_rna(X).astype(np.float64) @ tf32_rna(Wg).astype(np.float64).T
    Ut = tf32_rna(X).astype(np.float64) @ tf32_rna(Wu).astype(np.float64).T
    err_plain = np.abs(silu_mul(Gt, Ut) - ref["H"])
    assert np.mean(err_plain > b) > 0.2   # most outputs violate the bound

    xh, xl = split(X)
    gh, gl = split(Wg)
    uh, ul = split(Wu)
    G3 = xh @ gh.T + xh @ gl.T + xl @ gh.T
    U3 = xh @ uh.T + xh @ ul.T + xl @ uh.T
    err3 = np.abs(silu_mul(G3, U3) - ref["H"])
    assert np.all(err3 <= 0.05 * b)       # with a wide margin for fp32 sums
