"""swiglu_bwd_dx_noalloc: dX of the projection's backward without any device
allocation, for callers that cannot allocate while they run (for instance a
loop that handed all device memory to its own allocator at start-up).  It
keeps the split tail's partial tiles in a fixed array inside the library
instead of a workspace from the memory pool, and must give exactly what
swiglu_bwd_dx gives.

Two calls go back to back on one stream -- the second reuses the array the
first left filled, with another shape and split -- and each output is
checked against swiglu_bwd_dx on the same inputs.  The file sorts last so
that a run stopping at its first failure has run every other test first."""
import numpy as np
import pytest
import torch

from gpu_util import dev, f64
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu


def _inputs(M, K, N, dtype, seed):
    Wg = synth.normal((N, K), seed, 1.0 / np.sqrt(K), dtype)
    Wu = synth.normal((N, K), seed + 1, 1.0 / np.sqrt(K), dtype)
    dG = synth.normal((M, N), seed + 2, 1.0, dtype)
    dU = synth.normal((M, N), seed + 3, 1.0, dtype)
    return [t.to(dev()) for t in (dG, dU, Wg, Wu)]


def _call(name, d, M, K, N, dtype, stream):
    code = _capi.SWIGLU_FP32 if dtype == "f32" else _capi.SWIGLU_BF16
    dX = torch.empty((M, K), dtype=d[0].dtype, device=d[0].device)
    st = getattr(_capi.lib(), name)(d[0].data_ptr(), d[1].data_ptr(), d[2].data_ptr(),
                                    d[3].data_ptr(), dX.data_ptr(), M, K, N, code,
                                    stream.cuda_stream)
    assert st == 0, _capi.status_string(st)
    return dX


# (M, K, N, dtype): with 148 SMs, 1280 x 4096 splits 12 tail tiles 8 ways
# (12.6 MB of partials), 300 x 520 splits 9 tiles of 128 columns 2 ways; the
# bf16 case takes no scratch.
CASES = [[(1280, 4096, 1024, "f32"), (300, 520, 200, "f32")],
         [(256, 512, 2048, "f32"), (130, 264, 136, "bf16")]]


@pytest.mark.parametrize("pair", CASES, ids=["split_then_split", "split_then_bf16"])
def test_noalloc_bwd_dx_matches_swiglu_bwd_dx(pair):
    stream = torch.cuda.current_stream()
    data = [_inputs(M, K, N, dt, seed=100 + 7 * i) for i, (M, K, N, dt) in enumerate(pair)]
    got = [_call("swiglu_bwd_dx_noalloc", d, *shape, stream) for d, shape in zip(data, pair)]
    assert _capi.swiglu_sync_status() == 0
    for d, shape, out in zip(data, pair, got):
        M, K, N, dt = shape
        ref = _call("swiglu_bwd_dx", d, *shape, stream)
        assert _capi.swiglu_sync_status() == 0
        a, b = f64(out), f64(ref)
        if dt == "f32":
            # the fp32 tests' bound, relative to the magnitudes summed
            g, u, wg, wu = (f64(t) for t in d)
            mag = np.abs(g) @ np.abs(wg) + np.abs(u) @ np.abs(wu)
            assert np.all(np.abs(a - b) <= 1e-5 * (mag + np.abs(b)) + 1e-30)
        else:
            assert np.all(np.abs(a - b) <= 1e-2 * np.abs(b) + 1e-3)
        # the same plan and the same arithmetic: identical bits
        assert torch.equal(out, ref)
