"""The TTQ linear layer sharded along its output rows d' over the ranks of
a torch.distributed process group: each rank quantises and multiplies its
own rows of W (and of the low-rank B), and the output columns are gathered.

Every output row of the layer depends on one row of W only (the statistic D
comes from the full X, which every rank holds, and the quantiser's groups
run along the input channels of one row), so the shards need no exchange
before the product; the one collective is the all-gather of Y.  Each rank
computes D itself (O(dT) work, small against the O(d'd) quantiser).

The local compute is `ttq.ttq_linear_forward` (the CUDA path); the
all-gather goes through the process group's backend (NCCL over NVLink on
the GPU, gloo in the CPU tests, which pass their own `local_forward`).
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def shard_rows(dp: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [start, stop) of a d' = dp output dimension that rank `rank` of
    `world` owns: contiguous slices of a multiple of 8 rows (so that each
    rank's Y rows stay 16-byte strided in bf16), the last one ragged."""
    if world < 1 or not 0 <= rank < world or dp < 0:
        raise ValueError("bad shard request")
    per = -(-dp // world)
    per = -(-per // 8) * 8
    start = min(rank * per, dp)
    return start, min(start + per, dp)


def linear_forward_sharded(X: torch.Tensor, W_local: torch.Tensor, A: torch.Tensor | None,
                           B_local: torch.Tensor | None, p: float, lam: float, alpha: float,
                           bits: int, group: int, dp: int, pg=None,
                           local_forward: Callable | None = None, **kwargs) -> torch.Tensor:
    """Y [T][dp] of the layer whose rows this rank holds as W_local (and
    B_local), with the rows of W split as `shard_rows(dp, world, rank)`.

    local_forward(X, W_local, A, B_local, p, lam, alpha, bits, group, **kwargs)
    returns this rank's Y columns [T][rows]; by default the CUDA forward.
    """
    world = dist.get_world_size(pg)
    rank = dist.get_rank(pg)
    start, stop = shard_rows(dp, world, rank)
    if W_local.shape[0] != stop - start:
        raise ValueError(f"rank {rank} holds {W_local.shape[0]} rows of W, expected {stop - start}")
    if local_forward is None:
        from test_weight_quantization_ttq_b200 import ttq
        local_forward = ttq.ttq_linear_forward
    T = X.shape[0]
    Y_local = local_forward(X, W_local, A, B_local, p, lam, alpha, bits, group, **kwargs)
    per = shard_rows(dp, world, 0)[1]  # the widest shard
    # every rank contributes a [T][per] block (its columns, zero padded)
    send = torch.zeros((T, per), dtype=Y_local.dtype, device=Y_local.device)
    send[:, : stop - start] = Y_local
    blocks = [torch.empty_like(send) for _ in range(world)]
    dist.all_gather(blocks, send, group=pg)
    cols = []
    for r in range(world):
        a, b = shard_rows(dp, world, r)
        cols.append(blocks[r][:, : b - a])
    return torch.cat(cols, dim=1)
