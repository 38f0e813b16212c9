"""C-ABI behaviour on a GPU: degenerate sizes, error codes with real device
pointers, and that each route's kernel is the one that ran."""
import pytest
import torch

from gpu_util import dev
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu


def test_k_zero_writes_zeros():
    H = torch.full((5, 16), 7.0, dtype=torch.bfloat16, device=dev())
    X = torch.empty((5, 0), dtype=torch.bfloat16, device=dev())
    W = torch.empty((16, 0), dtype=torch.bfloat16, device=dev())
    _capi.swiglu_fwd(X, W, W, H)
    assert _capi.swiglu_sync_status() == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_ZERO_K
    assert bool((H == 0).all())


def test_empty_problems_are_noops():
    lib = _capi.lib()
    s = torch.cuda.current_stream().cuda_stream
    assert lib.swiglu_fwd(None, None, None, None, 0, 64, 64, 0, s) == 0
    assert _capi.swiglu_last_route() == _capi.ROUTE_NONE
    assert lib.swiglu_fwd(None, None, None, None, 4, 64, 0, 0, s) == 0
    assert lib.dswiglu_bwd(None, None, None, None, None, 0, s) == 0


def test_error_codes_with_device_pointers():
    lib = _capi.lib()
    s = torch.cuda.current_stream().cuda_stream
    X, Wg, Wu = (t.to(dev()) for t in synth.swiglu_inputs(4, 64, 64, "bf16"))
    H = torch.empty((4, 64), dtype=torch.bfloat16, device=dev())
    p = (X.data_ptr(), Wg.data_ptr(), Wu.data_ptr(), H.data_ptr())
    assert lib.swiglu_fwd(*p, 4, 64, 64, 0, s) == 0
    assert lib.swiglu_fwd(p[0] + 2, *p[1:], 4, 64, 64, 0, s) == _capi.SWIGLU_ERR_MISALIGNED_PTR
    assert lib.swiglu_fwd(*p, 4, 60, 64, 0, s) == _capi.SWIGLU_ERR_MISALIGNED_DIM
    assert lib.swiglu_fwd(*p, 4, 64, 64, 7, s) == _capi.SWIGLU_ERR_BAD_DTYPE
    assert lib.swiglu_fwd(*p, -1, 64, 64, 0, s) == _capi.SWIGLU_ERR_BAD_DIM
    assert lib.swiglu_fwd(p[0], p[1], p[2], p[0], 4, 64, 64, 0, s) == _capi.SWIGLU_ERR_OVERLAP
    assert lib.swiglu_fwd(p[0], None, p[2], p[3], 4, 64, 64, 0, s) == _capi.SWIGLU_ERR_NULL_POINTER
    assert _capi.swiglu_sync_status() == 0


def test_routes_engage_their_kernels():
    for M, route in ((1, _capi.ROUTE_DECODE_BF16), (8, _capi.ROUTE_DECODE_BF16),
                     (9, _capi.ROUTE_STREAM_TC_BF16), (128, _capi.ROUTE_STREAM_TC_BF16),
                     (129, _capi.ROUTE_GEMM_BF16), (200, _capi.ROUTE_GEMM_BF16)):
        X, Wg, Wu = (t.to(dev()) for t in synth.swiglu_inputs(M, 128, 64, "bf16"))
        _capi.swiglu_fwd(X, Wg, Wu)
        assert _capi.swiglu_last_route() == route, M
    assert _capi.swiglu_sync_status() == 0


def test_rank3_input_is_flattened():
    X, Wg, Wu = synth.swiglu_inputs(6, 64, 32, "bf16", seed=2)
    Xd, Wgd, Wud = (t.to(dev()) for t in (X, Wg, Wu))
    flat = _capi.swiglu_fwd(Xd, Wgd, Wud)
    H3 = _capi.swiglu_fwd(Xd.view(2, 3, 64), Wgd, Wud)
    assert H3.shape == (2, 3, 32)
    assert torch.equal(H3.reshape(6, 32), flat)


def test_bounded_wait_timeout_is_reported_and_recoverable():
    """The failure path without a fault: a wait that nothing completes gives
    up after ~1 ms, the host reads SWIGLU_ERR_TIMEOUT once, and the context
    keeps working."""
    import torch
    from up_projection_b200 import _capi
    s = torch.cuda.current_stream().cuda_stream
    assert _capi.swiglu_sync_status() == 0
    assert _capi.lib().swiglu_selftest_wait_timeout(s) == 0
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_ERR_TIMEOUT
    assert _capi.swiglu_sync_status() == 0          # the word was cleared
    X = torch.randn(130, 64, device="cuda").to(torch.bfloat16)
    W = (torch.randn(64, 64, device="cuda") / 8).to(torch.bfloat16)
    H = _capi.swiglu_fwd(X, W, W)
    assert _capi.swiglu_sync_status() == 0 and bool(torch.isfinite(H.float()).all())


@pytest.mark.parametrize("nbytes", [16, 12288, 12288 * 7 + 48, 6912 * 1536 * 2])
def test_read_floor_reads_every_byte_once(nbytes):
    """The bench's pure-read probe: every CTA folds words 0 and 3 of each
    16-byte vector it read into its sink word, so the XOR of all sink words is
    the XOR of those words over both buffers -- each byte read exactly once
    (a chunk read twice or skipped changes it)."""
    import numpy as np
    g = torch.Generator(device="cpu").manual_seed(nbytes)
    A = torch.randint(0, 2 ** 31 - 1, (nbytes // 4,), generator=g, dtype=torch.int32)
    B = torch.randint(0, 2 ** 31 - 1, (nbytes // 4,), generator=g, dtype=torch.int32)
    sink = torch.zeros(int(_capi.lib().swiglu_read_floor_sink_words()), dtype=torch.int32,
                       device=dev())
    _capi.swiglu_read_floor(A.to(dev()), B.to(dev()), sink)
    torch.cuda.synchronize()
    got = np.bitwise_xor.reduce(sink.cpu().numpy().view(np.uint32))
    want = np.uint32(0)
    for t in (A, B):
        v = t.numpy().view(np.uint32).reshape(-1, 4)
        want ^= np.bitwise_xor.reduce(v[:, 0]) ^ np.bitwise_xor.reduce(v[:, 3])
    assert int(got) == int(want)
