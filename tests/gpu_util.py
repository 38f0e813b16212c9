"""Shared helpers of the GPU parity tests: device transfer, the tolerance
checks the tests assert, sampling of full-size outputs, guard canaries."""
from __future__ import annotations

import numpy as np
import torch

# bf16 outputs with fp32 accumulation: |gpu - ref| <= 1e-2 |ref| + 1e-3.
BF16_RTOL = 1e-2
BF16_ATOL = 1e-3
# fp32-input mode: 1e-5 of the size of the terms before cancellation.
FP32_FWD_TOL = 1e-5
# fp32 dSwiGLU: 1e-6 of the size of the terms before cancellation.
FP32_BWD_TOL = 1e-6


def fp32_bound(G, U, H, AG, AU):
    """Per-element bound of the fp32-input mode: 1e-5 of the size of the terms
    before cancellation, propagated through h = silu(g) u (AG, AU: the sums of
    |x w| behind G and U)."""
    s = 1.0 / (1.0 + np.exp(-np.clip(G, -700, 700)))
    silu = G * s
    dsilu = s * (1.0 + G * (1.0 - s))
    return FP32_FWD_TOL * (np.abs(H) + np.abs(silu) * AU + np.abs(U) * np.abs(dsilu) * AG) + 1e-30


def dev():
    return torch.device("cuda:0")


def to_dev(*ts):
    return tuple(t.to(dev()) for t in ts)


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def assert_bf16_close(gpu: np.ndarray, ref: np.ndarray, what: str):
    gpu = np.asarray(gpu, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert gpu.shape == ref.shape
    bound = BF16_RTOL * np.abs(ref) + BF16_ATOL
    err = np.abs(gpu - ref)
    bad = ~(err <= bound)
    if bad.any():
        i = np.flatnonzero(bad)
        raise AssertionError(
            f"{what}: {bad.sum()} of {gpu.size} outside |d| <= 1e-2|ref| + 1e-3; "
            f"first at {i[:5].tolist()}: gpu={gpu[i[:5]].tolist()} ref={ref[i[:5]].tolist()}")


def assert_within(err: np.ndarray, bound: np.ndarray, what: str):
    err = np.asarray(err, dtype=np.float64).ravel()
    bound = np.asarray(bound, dtype=np.float64).ravel()
    bad = ~(err <= bound)
    if bad.any():
        i = np.flatnonzero(bad)
        ratio = err[i] / np.maximum(bound[i], 1e-300)
        raise AssertionError(f"{what}: {bad.sum()} of {err.size} outside bound; "
                             f"first at {i[:5].tolist()}, err/bound={ratio[:5].tolist()}")


def sample_indices(M: int, N: int, count: int, seed: int = 1234):
    """Random output coordinates plus the four corners and tile edges."""
    r = np.random.Generator(np.random.PCG64(seed))
    im = r.integers(0, M, size=count)
    inn = r.integers(0, N, size=count)
    edge_m = np.array([0, M - 1, min(127, M - 1), min(128, M - 1), M - 1, 0])
    edge_n = np.array([0, N - 1, min(127, N - 1), min(128, N - 1), 0, N - 1])
    return np.concatenate([im, edge_m]), np.concatenate([inn, edge_n])


GUARD = 4096  # guard elements on each side of an output buffer


def guarded_empty(numel: int, dtype, fill: float = 1234.5):
    """An output buffer with canary regions before and after it.  Returns
    (full buffer, view of the numel payload).  The payload starts 16-byte
    aligned since GUARD * element size is a multiple of 16."""
    full = torch.full((numel + 2 * GUARD,), fill, dtype=dtype, device=dev())
    return full, full[GUARD:GUARD + numel]


def assert_guards_intact(full: torch.Tensor, fill: float = 1234.5):
    g0 = full[:GUARD]
    g1 = full[-GUARD:]
    assert bool((g0 == fill).all()) and bool((g1 == fill).all()), "output guard overwritten"


# Smallest magnitudes that round to infinity (round-to-nearest-even, no
# saturation): the midpoint between the largest finite value and 2^128.
BF16_OVERFLOW = 2.0 ** 128 - 2.0 ** 119
FP32_OVERFLOW = 2.0 ** 128 - 2.0 ** 103


def assert_ieee_close(gpu, ref, what: str, dtype: str = "bf16", bound=None):
    """Outputs that may hold NaN and infinities, against the fp64 reference:
    NaN exactly where the reference is NaN; the same signed infinity where the
    reference is infinite or rounds to infinity in the output type; finite
    elsewhere and within the tolerance (bf16: 1e-2 |ref| + 1e-3; fp32: the
    per-element `bound`).  Returns the count of each class."""
    gpu = np.asarray(gpu, dtype=np.float64).ravel()
    ref = np.asarray(ref, dtype=np.float64).ravel()
    assert gpu.shape == ref.shape
    over = BF16_OVERFLOW if dtype == "bf16" else FP32_OVERFLOW
    nan_r = np.isnan(ref)
    inf_r = ~nan_r & (np.abs(ref) >= over)
    fin_r = ~(nan_r | inf_r)
    bad = np.isnan(gpu) != nan_r
    if bad.any():
        i = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{what}: NaN positions differ ({int(bad.sum())}); first at "
                             f"{i.tolist()}: gpu={gpu[i].tolist()} ref={ref[i].tolist()}")
    want_inf = np.where(ref > 0, np.inf, -np.inf)
    bad = inf_r & (gpu != want_inf)
    if bad.any():
        i = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} infinities differ; first at "
                             f"{i.tolist()}: gpu={gpu[i].tolist()} ref={ref[i].tolist()}")
    bad = fin_r & ~np.isfinite(gpu)
    if bad.any():
        i = np.flatnonzero(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} non-finite where the reference is "
                             f"finite; first at {i.tolist()}: gpu={gpu[i].tolist()} "
                             f"ref={ref[i].tolist()}")
    if dtype == "bf16":
        assert_bf16_close(gpu[fin_r], ref[fin_r], what)
    else:
        b = np.asarray(bound, dtype=np.float64).ravel()[fin_r]
        assert_within(np.abs(gpu[fin_r] - ref[fin_r]), b, what)
    return {"nan": int(nan_r.sum()), "inf": int(inf_r.sum()), "finite": int(fin_r.sum())}
