"""Multi-rank host logic on CPU: world_size 2 (and 3) over gloo.

Covers the column split (shards are disjoint, aligned, cover N), the max
over ranks used for timing, and the one all-gather a full-H consumer pays.
The per-rank shard values come from the oracle (this is a test of the
plumbing, not of a kernel)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from up_projection_b200 import parallel


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    try:
        import datetime
        dist.init_process_group("gloo", rank=rank, world_size=world,
                                timeout=datetime.timedelta(seconds=60))
        import oracle
        from up_projection_b200 import synth
        M, K, N = 3, 64, 136
        X, Wg, Wu = synth.swiglu_inputs(M, K, N, "bf16", seed=4)
        Wg_s, Wu_s = parallel.shard_weights(Wg, Wu, world, rank)
        H_s = torch.from_numpy(oracle.swiglu_fwd(X, Wg_s, Wu_s, "bf16")["H"])
        H = parallel.gather_columns(H_s, N)
        full = oracle.swiglu_fwd(X, Wg, Wu, "bf16")["H"]
        ok_gather = bool(np.array_equal(H.numpy(), full))
        mx = parallel.max_over_ranks(10.0 + rank)
        q.put((rank, ok_gather, mx))
        dist.barrier()
        dist.destroy_process_group()
    except Exception as exc:  # report to the parent instead of hanging it
        q.put((rank, repr(exc), None))


@pytest.mark.parametrize("world", [2, 3])
def test_column_split_gather_and_max(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, mx in results:
        assert ok is True, (rank, ok)
        assert mx == 10.0 + world - 1


def test_column_shard_partition():
    for N in (8, 64, 136, 6912, 14336):
        for world in (1, 2, 3, 4, 8):
            bounds = [parallel.column_shard(N, world, r) for r in range(world)]
            assert bounds[0][0] == 0 and bounds[-1][1] == N
            for (a0, a1), (b0, b1) in zip(bounds, bounds[1:]):
                assert a1 == b0
            for a0, a1 in bounds:
                assert a0 % 8 == 0 and a1 % 8 == 0 and a1 >= a0
            sizes = [b - a for a, b in bounds]
            assert max(sizes) - min(sizes) <= 8
    with pytest.raises(ValueError):
        parallel.column_shard(12, 2, 0)
