"""Fused forward kernels (decode weight streaming, tcgen05 dual GEMM) vs the
fp64 oracle, through the C ABI: element by element on small and ragged
shapes, on sampled outputs at the full workload sizes, bit-exact on integer
inputs, with guard canaries around every output."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import (assert_bf16_close, assert_guards_intact, dev, f64, guarded_empty,
                      sample_indices, to_dev)
from up_projection_b200 import _capi, synth

pytestmark = pytest.mark.gpu


def run_fwd(X, Wg, Wu, expect_route=None):
    M, K = X.shape
    N = Wg.shape[0]
    Xd, Wgd, Wud = to_dev(X, Wg, Wu)
    full, H = guarded_empty(M * N, X.dtype)
    _capi.swiglu_fwd(Xd, Wgd, Wud, H.view(M, N))
    st = _capi.swiglu_sync_status()
    assert st == _capi.SWIGLU_OK, _capi.status_string(st)
    if expect_route is not None:
        assert _capi.swiglu_last_route() == expect_route
    assert_guards_intact(full)
    return H.view(M, N).cpu()


def check_full(X, Wg, Wu, expect_route, what):
    H = run_fwd(X, Wg, Wu, expect_route)
    ref = oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"]
    assert_bf16_close(f64(H), ref, what)
    return H


# ---------------------------------------------------------------- decode

def test_tiny_config():
    """X bf16 [4, 256], Wg/Wu [512, 256] ~ N(0, 1/K), seed 0."""
    X, Wg, Wu = synth.swiglu_inputs(4, 256, 512, "bf16", seed=0)
    check_full(X, Wg, Wu, _capi.ROUTE_DECODE_BF16, "tiny")


@pytest.mark.parametrize("M", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("K,N", [(256, 512), (264, 72), (8, 8), (1536, 6912), (40, 1032),
                                 (5000, 264)])
def test_decode_shapes(M, K, N):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 1000 + K)
    check_full(X, Wg, Wu, _capi.ROUTE_DECODE_BF16, f"decode M={M} K={K} N={N}")


@pytest.mark.parametrize("M", [1, 2, 4, 8])
def test_decode_llama7b_full(M):
    """LLaMA-2 7B up/gate shape: K = 4096, N = 11008 (all outputs checked)."""
    X, Wg, Wu = synth.swiglu_inputs(M, 4096, 11008, "bf16", seed=7 + M)
    check_full(X, Wg, Wu, _capi.ROUTE_DECODE_BF16, f"llama7b M={M}")


@pytest.mark.parametrize("M", [9, 16, 17, 31, 64, 128])
@pytest.mark.parametrize("K,N", [(264, 72), (8, 8), (40, 1032), (2000, 264), (520, 6912)])
def test_small_m_gemm_shapes(M, K, N):
    """9 <= M <= 128 with K not a multiple of 64 takes the dual GEMM (one
    ragged M tile); every output against the oracle."""
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 1000 + K + 1)
    check_full(X, Wg, Wu, _capi.ROUTE_GEMM_BF16, f"gemm M={M} K={K} N={N}")


# ------------------------------------------------- tcgen05 weight stream

@pytest.mark.parametrize("M", [9, 15, 16, 17, 24, 32, 33, 47, 64, 65, 100, 127, 128])
@pytest.mark.parametrize("K,N", [(64, 8), (128, 520), (256, 512), (1536, 6912), (832, 1032),
                                 (4096, 264)])
def test_stream_tc_shapes(M, K, N):
    """9 <= M <= 128, K a multiple of 64: one k-block (K = 64), a partial last
    slice (K = 832), several slices, ragged M against the 8-row X boxes;
    every output against the oracle."""
    assert _capi.swiglu_route_for(M, K, N, 0) == _capi.ROUTE_STREAM_TC_BF16
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 977 + K + N)
    check_full(X, Wg, Wu, _capi.ROUTE_STREAM_TC_BF16, f"stream M={M} K={K} N={N}")


@pytest.mark.parametrize("M", [16, 32, 64])
def test_stream_tc_llama7b_full(M):
    """LLaMA-2 7B up/gate shape at batched-decode M (all outputs checked)."""
    X, Wg, Wu = synth.swiglu_inputs(M, 4096, 11008, "bf16", seed=70 + M)
    check_full(X, Wg, Wu, _capi.ROUTE_STREAM_TC_BF16, f"llama7b M={M}")


def test_stream_tc_many_units_per_cta():
    """N = 8 * 148 * 32 + 8: more units than TMEM holds for one CTA per SM,
    so the grid grows past the SM count; sampled outputs incl. the last."""
    M, K, N = 24, 128, 8 * 148 * 32 + 8
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=5)
    H = run_fwd(X, Wg, Wu, _capi.ROUTE_STREAM_TC_BF16)
    im, inn = sample_indices(M, N, 6000)
    im = np.concatenate([im, np.arange(M)])
    inn = np.concatenate([inn, np.full(M, N - 1)])
    ref = oracle.swiglu_fwd_points(X, Wg, Wu, im, inn, "bf16")["H"]
    assert_bf16_close(f64(H[im, inn]), ref, "stream many units")


@pytest.mark.parametrize("layout", ["same", "halves", "halves_swapped", "far"])
def test_stream_tc_weight_layouts(layout):
    """The gate and up rows come through one 4-D view whose matrix stride is
    the distance between the buffers (either order), or, for Wg == Wu,
    through two 3-D views: same results in every layout."""
    M, K, N = 24, 512, 1032
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=31)
    if layout == "same":
        Wu = Wg
    both = torch.stack([Wg, Wu]).to(dev())
    if layout == "same":
        Wgd = Wud = both[0]
    elif layout == "halves":
        Wgd, Wud = both[0], both[1]
    elif layout == "halves_swapped":
        both = torch.stack([Wu, Wg]).to(dev())
        Wgd, Wud = both[1], both[0]
    else:  # separate allocations with a large buffer between them
        Wgd = Wg.to(dev())
        gap = torch.empty(64 << 20, dtype=torch.uint8, device=dev())
        Wud = Wu.to(dev())
        del gap
    Xd = X.to(dev())
    H = _capi.swiglu_fwd(Xd, Wgd, Wud)
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert _capi.swiglu_last_route() == _capi.ROUTE_STREAM_TC_BF16
    assert_bf16_close(f64(H), oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"], f"stream layout {layout}")


def test_stream_tc_deterministic():
    X, Wg, Wu = synth.swiglu_inputs(32, 1536, 6912, "bf16", seed=4)
    a = run_fwd(X, Wg, Wu, _capi.ROUTE_STREAM_TC_BF16)
    b = run_fwd(X, Wg, Wu, _capi.ROUTE_STREAM_TC_BF16)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_small_m_integer_exact():
    """Integer operands with every gate pre-activation >= 17: sigmoid rounds
    to 1 in fp32, so H = bf16_rne(fp32(G * U)) exactly, for every tile and
    lane position -- any indexing or layout slip changes bits.  Covers the
    decode kernel, the tcgen05 weight stream and the dual GEMM at small M."""
    routes = set()
    for M, K, N in [(8, 256, 512), (3, 136, 1024), (1, 64, 8), (9, 264, 512), (32, 136, 1024),
                    (17, 72, 8), (9, 256, 512), (64, 128, 1032), (128, 192, 264), (33, 1536, 264),
                    (17, 64, 8), (65, 256, 136)]:
        X, Wg, Wu = synth.integer_inputs(M, K, N, seed=M + K)
        H = run_fwd(X, Wg, Wu)
        routes.add(_capi.swiglu_last_route())
        G = X.to(torch.float64) @ Wg.to(torch.float64).T
        U = X.to(torch.float64) @ Wu.to(torch.float64).T
        assert float(G.min()) >= 17.0
        expect = (G * U).to(torch.float32).to(torch.bfloat16)
        assert torch.equal(H.view(torch.int16), expect.view(torch.int16)), (M, K, N)
    assert routes == {_capi.ROUTE_DECODE_BF16, _capi.ROUTE_STREAM_TC_BF16, _capi.ROUTE_GEMM_BF16}


def test_decode_deterministic():
    X, Wg, Wu = synth.swiglu_inputs(8, 1536, 6912, "bf16", seed=3)
    a = run_fwd(X, Wg, Wu)
    b = run_fwd(X, Wg, Wu)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


# --------------------------------------------------------------- dual GEMM

@pytest.mark.parametrize("M,K,N", [
    (129, 256, 512),     # smallest GEMM-route M at K a multiple of 64
    (33, 264, 512),      # smallest GEMM-route M at other K
    (9, 65544, 64),      # K not a multiple of 64, X rows too large for decode
    (129, 64, 128),      # one N tile, one k-block, a one-row second M tile
    (200, 128, 256),     # two k-blocks, two N tiles
    (129, 72, 136),      # ragged M, ragged K (not a multiple of 64), ragged N
    (300, 520, 392),     # several ragged tiles
    (256, 4096, 512),    # long K: the smem ring wraps many times
])
def test_gemm_small_shapes(M, K, N):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M + K + N)
    check_full(X, Wg, Wu, _capi.ROUTE_GEMM_BF16, f"gemm M={M} K={K} N={N}")


def test_gemm_many_tiles_per_cta():
    """Enough tiles that every persistent CTA runs many, so both TMEM
    accumulator buffers and all smem stages are recycled."""
    M, K, N = 2048, 512, 4096
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=11)
    check_full(X, Wg, Wu, _capi.ROUTE_GEMM_BF16, "gemm many tiles")


def test_gemm_integer_exact():
    # M > 128 runs the pair form (256-row tiles over two SMs): a partly
    # empty second half (130), one full pair (256), several pairs (520)
    for M, K, N in [(256, 256, 384), (130, 64, 136), (520, 64, 264)]:
        X, Wg, Wu = synth.integer_inputs(M, K, N, seed=M + N)
        H = run_fwd(X, Wg, Wu, _capi.ROUTE_GEMM_BF16)
        G = X.to(torch.float64) @ Wg.to(torch.float64).T
        U = X.to(torch.float64) @ Wu.to(torch.float64).T
        assert float(G.min()) >= 17.0
        expect = (G * U).to(torch.float32).to(torch.bfloat16)
        diff = (H.view(torch.int16) != expect.view(torch.int16))
        assert not bool(diff.any()), f"{int(diff.sum())} mismatches, first {diff.nonzero()[:5].tolist()}"


def test_prefill_full_size_sampled():
    """LLaMA-3 8B prefill shape, the launch the bench times: M = 8192,
    K = 4096, N = 14336; sampled outputs against the oracle, plus a rerun
    that must be bitwise identical."""
    M, K, N = 8192, 4096, 14336
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=0)
    H = run_fwd(X, Wg, Wu, _capi.ROUTE_GEMM_BF16)
    im, inn = sample_indices(M, N, 4000)
    ref = oracle.swiglu_fwd_points(X, Wg, Wu, im, inn, "bf16")["H"]
    assert_bf16_close(f64(H[im, inn]), ref, "prefill sampled")
    # whole rows/columns at tile boundaries
    for m in (0, 127, 128, 8191):
        cols = np.arange(N)
        r = oracle.swiglu_fwd_points(X, Wg, Wu, np.full(N, m), cols, "bf16")["H"]
        assert_bf16_close(f64(H[m]), r, f"prefill row {m}")
    H2 = run_fwd(X, Wg, Wu)
    assert torch.equal(H.view(torch.int16), H2.view(torch.int16))


def test_decode_astrai_full_size_rotated_copies():
    """AstrAI-1B decode as the bench runs it: 16 rotated weight copies,
    M in {1, 2, 4, 8}; every output of copies 0 and 15 checked."""
    K, N, R = 1536, 6912, 16
    X8, Wg, Wu = synth.swiglu_inputs(8, K, N, "bf16", seed=0)
    Wgd = torch.empty((R, N, K), dtype=torch.bfloat16, device=dev())
    Wud = torch.empty_like(Wgd)
    Wgd[:] = Wg.to(dev())
    Wud[:] = Wu.to(dev())
    for M in (1, 2, 4, 8):
        X = X8[:M].contiguous()
        ref = oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"]
        Xd = X.to(dev())
        for r in (0, R - 1):
            H = _capi.swiglu_fwd(Xd, Wgd[r], Wud[r])
            assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
            assert _capi.swiglu_last_route() == _capi.ROUTE_DECODE_BF16
            assert_bf16_close(f64(H), ref, f"astrai M={M} copy={r}")


@pytest.mark.parametrize("K,N", [(1536, 6912), (4096, 11008), (256, 512), (5000, 264),
                                 (8, 8), (264, 72)])
def test_decode_weights_stable_path(K, N):
    """The programmatic-dependent-launch path (weights prefetched before the
    preceding kernel finishes) gives oracle-exact-within-tolerance results;
    at large K and M < 8 this is also the compact X layout (only the M rows
    of X staged, the other rows of the MMA operand zero in registers)."""
    for M in (1, 2, 3, 5, 8):
        X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M + 5)
        Xd, Wgd, Wud = to_dev(X, Wg, Wu)
        H = _capi.swiglu_fwd(Xd, Wgd, Wud, weights_stable=True)
        assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
        assert _capi.swiglu_last_route() == _capi.ROUTE_DECODE_BF16
        assert_bf16_close(f64(H), oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"], f"pdl M={M} K={K}")


@pytest.mark.parametrize("K,N", [(1536, 6912), (4096, 11008), (256, 512), (264, 72)])
def test_decode_weights_stable_mid_m(K, N):
    """weights_stable at 9 <= M <= 32 on the route the shape takes: the
    tcgen05 weight stream (its first stages' weights requested before the
    wait for X), or the dual GEMM where K is not a multiple of 64."""
    for M in (9, 16, 24, 32):
        X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M + 9)
        Xd, Wgd, Wud = to_dev(X, Wg, Wu)
        H = _capi.swiglu_fwd(Xd, Wgd, Wud, weights_stable=True)
        assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
        assert _capi.swiglu_last_route() == _capi.swiglu_route_for(M, K, N, 0)
        assert_bf16_close(f64(H), oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"], f"pdl M={M} K={K}")


def test_decode_weights_stable_chain_reads_x_after_producer():
    """A chain of dependent decode calls on one stream, each call's input X
    being the previous call's output H, all with weights_stable: every X read
    must see the finished output of the call before it."""
    K = N = 1536
    M, steps = 8, 12
    X0, _, _ = synth.swiglu_inputs(M, K, N, "bf16", seed=21)
    Ws = [synth.swiglu_inputs(1, K, N, "bf16", seed=100 + i)[1:] for i in range(steps)]
    dev_ws = [(g.to(dev()), u.to(dev())) for g, u in Ws]
    x = X0.to(dev())
    outs = []
    for g, u in dev_ws:
        x = _capi.swiglu_fwd(x, g, u, weights_stable=True)
        outs.append(x)
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    # step by step on the host: each oracle step takes the GPU's previous
    # (bf16) output, so errors do not compound across the chain
    prev = X0
    for i, (g, u) in enumerate(Ws):
        ref = oracle.swiglu_fwd(prev, g, u, "bf16")["H"]
        got = outs[i].cpu()
        assert_bf16_close(f64(got), ref, f"chain step {i}")
        prev = got


def _random_shapes(seed, count, ms):
    r = np.random.Generator(np.random.PCG64(seed))
    out = []
    for i in range(count):
        M = int(ms[i % len(ms)])
        K = int(r.integers(1, 80)) * 8
        N = int(r.integers(1, 80)) * 8
        out.append((M, K, N))
    return out


@pytest.mark.parametrize("M,K,N", _random_shapes(2024, 16, [129, 130, 160, 200, 255, 257, 300, 511]))
def test_gemm_random_odd_shapes(M, K, N):
    """Seeded random shapes around tile boundaries: ragged M (127, 129, 257...),
    K and N any multiple of 8 up to 632, every output against the oracle."""
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 7 + K * 3 + N)
    check_full(X, Wg, Wu, _capi.ROUTE_GEMM_BF16, f"gemm M={M} K={K} N={N}")


@pytest.mark.parametrize("M,K,N", _random_shapes(2025, 10, [1, 2, 3, 5, 7, 8])
                         + _random_shapes(2026, 10, [9, 11, 15, 19, 23, 28, 32]))
def test_decode_random_odd_shapes(M, K, N):
    """Random shapes at M <= 32 (decode at M <= 8; above, the tcgen05 stream
    where K is a multiple of 64, the dual GEMM otherwise)."""
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 11 + K * 5 + N)
    route = _capi.swiglu_route_for(M, K, N, 0)
    assert route == _capi.ROUTE_DECODE_BF16 if M <= 8 else route in (
        _capi.ROUTE_STREAM_TC_BF16, _capi.ROUTE_GEMM_BF16)
    check_full(X, Wg, Wu, route, f"small-M M={M} K={K} N={N}")


def _random_stream_shapes(seed, count):
    r = np.random.Generator(np.random.PCG64(seed))
    return [(int(r.integers(9, 129)), int(r.integers(1, 40)) * 64, int(r.integers(1, 200)) * 8)
            for _ in range(count)]


@pytest.mark.parametrize("M,K,N", _random_stream_shapes(2027, 16))
def test_stream_tc_random_shapes(M, K, N):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=M * 13 + K * 7 + N)
    check_full(X, Wg, Wu, _capi.ROUTE_STREAM_TC_BF16, f"stream M={M} K={K} N={N}")


@pytest.mark.parametrize("M", [16, 64, 128])
def test_stream_weights_stable_chain_reads_x_after_producer(M):
    """The tcgen05 weight stream under weights_stable requests its first
    stages' weights before waiting for the preceding grid and X only after
    it: a chain of dependent calls, each call's X the previous call's H
    (K = N, a multiple of 64), must see every finished output."""
    K = N = 512
    steps = 8
    X0, _, _ = synth.swiglu_inputs(M, K, N, "bf16", seed=23 + M)
    Ws = [synth.swiglu_inputs(1, K, N, "bf16", seed=200 + i)[1:] for i in range(steps)]
    dev_ws = [(g.to(dev()), u.to(dev())) for g, u in Ws]
    assert _capi.swiglu_route_for(M, K, N, 0) == _capi.ROUTE_STREAM_TC_BF16
    x = X0.to(dev())
    outs = []
    for g, u in dev_ws:
        x = _capi.swiglu_fwd(x, g, u, weights_stable=True)
        outs.append(x)
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert _capi.swiglu_last_route() == _capi.ROUTE_STREAM_TC_BF16
    prev = X0
    for i, (g, u) in enumerate(Ws):
        got = outs[i].cpu()
        assert_bf16_close(f64(got), oracle.swiglu_fwd(prev, g, u, "bf16")["H"], f"chain M={M} {i}")
        prev = got


def test_mixed_route_chain_weights_stable():
    """Decode and tcgen05-stream calls interleaved on one stream through two
    buffers: each call reads rows another call just wrote (read after write)
    and writes rows another call just read (write after read).  The chain
    runs once with plain stream ordering, checked step by step against the
    oracle, and once with weights_stable and nothing between the calls (so
    consecutive calls overlap under programmatic dependent launch); at
    K = N = 512 both launch forms sum in the same order, so the final
    buffers must agree bit for bit."""
    K = N = 512
    A0, _, _ = synth.swiglu_inputs(16, K, N, "bf16", seed=41)
    # (X buffer, rows), (H buffer, rows)
    plan = [(("A", 0, 16), ("B", 0, 16)),     # stream
            (("B", 0, 8), ("A", 0, 8)),       # decode; overwrites rows step 0 read
            (("A", 0, 16), ("B", 0, 16)),     # stream; rows 0..7 from step 1
            (("B", 8, 16), ("A", 8, 16)),     # decode
            (("A", 8, 16), ("B", 0, 8)),      # decode
            (("B", 0, 16), ("A", 0, 16)),     # stream
            (("A", 0, 8), ("B", 8, 16))]      # decode
    Ws = [synth.swiglu_inputs(1, K, N, "bf16", seed=300 + i)[1:] for i in range(len(plan))]
    dev_ws = [(g.to(dev()), u.to(dev())) for g, u in Ws]
    assert (_capi.swiglu_route_for(16, K, N, 0), _capi.swiglu_route_for(8, K, N, 0)) == \
        (_capi.ROUTE_STREAM_TC_BF16, _capi.ROUTE_DECODE_BF16)

    def run(ws, check):
        bufs = {"A": A0.to(dev()), "B": torch.zeros_like(A0, device=dev())}
        host = {"A": A0.clone(), "B": torch.zeros_like(A0)}
        for i, (((xn, x0, x1), (hn, h0, h1)), (g, u)) in enumerate(zip(plan, dev_ws)):
            _capi.swiglu_fwd(bufs[xn][x0:x1], g, u, bufs[hn][h0:h1], weights_stable=ws)
            if check:
                x = host[xn][x0:x1].clone()
                h = bufs[hn][h0:h1].cpu()
                assert_bf16_close(f64(h), oracle.swiglu_fwd(x, Ws[i][0], Ws[i][1], "bf16")["H"],
                                  f"mixed chain step {i}")
                host[hn][h0:h1] = h
        assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
        return bufs["A"].cpu(), bufs["B"].cpu()

    ref_a, ref_b = run(False, True)
    for _ in range(3):
        a, b = run(True, False)
        assert torch.equal(a.view(torch.int16), ref_a.view(torch.int16))
        assert torch.equal(b.view(torch.int16), ref_b.view(torch.int16))


@pytest.mark.parametrize("M", [65, 128])
def test_stream_tc_split_form_odd_units(M):
    """Wg == Wu takes the split form (two boxes, two MMAs per step); at MMA
    M = 128 its N is rounded up to 16 and an odd unit count per CTA reads 8
    rows past the box (accumulator columns never read).  N = 264: 33 units,
    one per CTA."""
    K, N = 512, 264
    X, Wg, _ = synth.swiglu_inputs(M, K, N, "bf16", seed=M + 77)
    Xd, Wgd = to_dev(X, Wg)
    H = _capi.swiglu_fwd(Xd, Wgd, Wgd)
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert _capi.swiglu_last_route() == _capi.ROUTE_STREAM_TC_BF16
    assert_bf16_close(f64(H), oracle.swiglu_fwd(X, Wg, Wg, "bf16")["H"], f"split M={M}")
    # distinct gate and up weights in the split form: a swap of the two
    # accumulator regions would change H (h(g, u) != h(u, g))
    X2, Wg2, Wu2 = synth.swiglu_inputs(M, K, N, "bf16", seed=M + 78)
    both = torch.stack([Wg2, Wu2]).to(dev())
    H2 = _capi.swiglu_fwd(X2.to(dev()), both[0], both[1])
    assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
    assert_bf16_close(f64(H2), oracle.swiglu_fwd(X2, Wg2, Wu2, "bf16")["H"], f"pair M={M}")
