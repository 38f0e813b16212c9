"""Multi-GPU plumbing for the fused SwiGLU projection (one process per GPU).

The op needs no collective on its data path: every output element depends on
one row of X and one row each of Wg and Wu, and SiLU acts per element.

* Row (M) split = data-parallel replicas: each rank runs its own tokens.
* Column (N) split = the column-parallel gate/up of tensor parallelism: rank
  r holds rows [n0, n1) of Wg and Wu (column_shard) and the full X, and
  writes H[:, n0:n1] with the same fused kernel -- the epilogue stays fused
  because silu(g) * u is per element.  A K split would be wrong for this op:
  partial G and U would need a reduction before the nonlinear epilogue.
* Only a consumer that needs the full H pays one all-gather along N
  (gather_columns), done by torch.distributed / NCCL.

Timing across ranks is the max over ranks (max_over_ranks)."""
from __future__ import annotations

import torch


def column_shard(N: int, world: int, rank: int, align: int = 8):
    """[n0, n1) of the N output columns owned by `rank`: contiguous, disjoint,
    covering [0, N), each boundary a multiple of `align` (so every shard is a
    valid 16-byte-aligned row block of bf16 weights), sizes differing by at
    most `align`."""
    if N % align != 0:
        raise ValueError(f"N={N} is not a multiple of {align}")
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    blocks = N // align
    b0 = blocks * rank // world
    b1 = blocks * (rank + 1) // world
    return b0 * align, b1 * align


def shard_weights(Wg: torch.Tensor, Wu: torch.Tensor, world: int, rank: int):
    """This rank's row blocks of Wg and Wu [N, K] (contiguous views)."""
    n0, n1 = column_shard(Wg.shape[0], world, rank)
    return Wg[n0:n1], Wu[n0:n1]


def max_over_ranks(x: float, group=None) -> float:
    """Max of a per-rank scalar (elapsed device time) over the group."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(x)
    device = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def gather_columns(H_shard: torch.Tensor, N: int, group=None) -> torch.Tensor:
    """Full H [M, N] from every rank's H[:, n0:n1] (one all-gather)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    M = H_shard.shape[0]
    widths = [column_shard(N, world, r)[1] - column_shard(N, world, r)[0] for r in range(world)]
    if H_shard.shape != (M, widths[rank]):
        raise ValueError("shard shape does not match column_shard")
    wmax = max(widths)
    pad = torch.zeros((M, wmax), dtype=H_shard.dtype, device=H_shard.device)
    pad[:, :widths[rank]] = H_shard
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:, :w] for p, w in zip(parts, widths)], dim=1)
