"""The column split of the multi-GPU plumbing run through the kernels on one
GPU: each rank's shard of the gate/up projection (rows [n0, n1) of Wg and
Wu, the column-parallel gate/up whose output TensorRT-LLM PR #17693 gathers
with gather_output) is one swiglu_fwd call on row-block views of the
weights.  Each shard's H is checked element by element against the oracle's
column slice, and the shards side by side against the unsharded call: every
route sums each output in an order that does not depend on N, so the
concatenation must equal it bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import FP32_FWD_TOL, assert_bf16_close, assert_within, dev, f64
from up_projection_b200 import _capi, parallel, synth

pytestmark = pytest.mark.gpu

CASES = [  # (id, M, K, N, dtype, route of the unsharded call)
    ("decode_m8", 8, 1536, 6912, "bf16", _capi.ROUTE_DECODE_BF16),
    ("stream_m32", 32, 1536, 6912, "bf16", _capi.ROUTE_STREAM_TC_BF16),
    ("gemm_m256", 256, 520, 2056, "bf16", _capi.ROUTE_GEMM_BF16),
    ("fp32_m130", 130, 264, 1032, "f32", _capi.ROUTE_GEMM_TF32X3),
]


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("cid,M,K,N,dtype,route", CASES, ids=[c[0] for c in CASES])
def test_column_shards_through_the_kernels(cid, M, K, N, dtype, route, world):
    X, Wg, Wu = synth.swiglu_inputs(M, K, N, dtype, seed=N + world)
    Xd, Wgd, Wud = (t.to(dev()) for t in (X, Wg, Wu))
    full = _capi.swiglu_fwd(Xd, Wgd, Wud)
    assert _capi.swiglu_last_route() == route
    ref = oracle.swiglu_fwd(X, Wg, Wu, dtype, want_magnitudes=(dtype == "f32"))
    shards = []
    for rank in range(world):
        n0, n1 = parallel.column_shard(N, world, rank)
        Wg_s, Wu_s = parallel.shard_weights(Wgd, Wud, world, rank)
        assert Wg_s.data_ptr() == Wgd.data_ptr() + n0 * K * Wgd.element_size()  # views
        H_s = _capi.swiglu_fwd(Xd, Wg_s, Wu_s)
        assert _capi.swiglu_sync_status() == _capi.SWIGLU_OK
        got = f64(H_s)
        want = ref["H"][:, n0:n1]
        if dtype == "bf16":
            assert_bf16_close(got, want, f"{cid} world={world} rank={rank}")
        else:
            G, U = ref["G"][:, n0:n1], ref["U"][:, n0:n1]
            s = 1.0 / (1.0 + np.exp(-np.clip(G, -700, 700)))
            bound = FP32_FWD_TOL * (np.abs(want) + np.abs(G * s) * ref["AU"][:, n0:n1]
                                    + np.abs(U) * np.abs(s * (1 + G * (1 - s)))
                                    * ref["AG"][:, n0:n1]) + 1e-30
            assert_within(np.abs(got - want), bound, f"{cid} world={world} rank={rank}")
        shards.append(H_s)
    cat = torch.cat(shards, dim=1)
    bits = torch.int16 if dtype == "bf16" else torch.int32
    assert torch.equal(cat.view(bits), full.view(bits))
