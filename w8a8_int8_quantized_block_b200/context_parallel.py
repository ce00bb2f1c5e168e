"""Token-sharded (context-parallel) linear over several GPUs.

Token rows are independent through the whole linear (rotation, rowwise
quantisation, GEMM and epilogue act on one row at a time), so a sequence can
be split across GPUs by rows with no exchange inside the path.  The pages run
their video pipeline with context parallelism across GPUs ("HyperFlow H3
Flash MLX", section "How to run": the --gpus option); when every GPU needs
the whole output afterwards, one all-gather of the bf16 rows follows (NCCL
over NVLink / NVSwitch).  That gather is the only data-path collective.

Each rank holds its own contiguous shard of the tokens (token_shard gives the
split).  Shards are padded to the longest one so that the gather moves equal
pieces; when the number of tokens divides evenly, the gathered buffer is the
output itself, otherwise the padding rows are dropped with one copy.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist


def token_shard(M: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [start, end) of the M tokens that `rank` of `world` holds: equal
    shards of ceil(M / world) rows, the last ones shorter (possibly empty)."""
    if M < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError("bad shard request")
    per = -(-M // world)
    start = min(M, rank * per)
    return start, min(M, start + per)


def linear_context_parallel(x_local: torch.Tensor, M: int, N: int, linear: Callable, *, group=None,
                            out: torch.Tensor | None = None) -> torch.Tensor:
    """y [M, N] on every rank, from this rank's token shard x_local [m_r, K].

    `linear(x, out)` computes the shard's rows into `out` (for the B200 path,
    a closure over convrot.linear_fused with the packed weights).  Every rank
    of `group` must call this with the same M and N, in the same order (the
    gather is a collective)."""
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    start, end = token_shard(M, world, rank)
    if x_local.shape[0] != end - start:
        raise ValueError(f"rank {rank} holds {x_local.shape[0]} rows, its shard is {end - start}")
    per = -(-M // world)
    even = per * world == M
    if world == 1:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x_local.device) if out is None else out
        if M:
            linear(x_local, y)
        return y
    gathered = out if (even and out is not None) else torch.empty((per * world, N), dtype=torch.bfloat16,
                                                                    device=x_local.device)
    mine = gathered[rank * per:(rank + 1) * per]  # this rank's piece, in place
    if end > start:
        linear(x_local, mine[:end - start])
    if end - start < per:
        mine[end - start:].zero_()  # padding rows: defined values on the wire
    dist.all_gather_into_tensor(gathered, mine, group=group)
    if even:
        return gathered
    y = torch.empty((M, N), dtype=torch.bfloat16, device=x_local.device) if out is None else out
    for r in range(world):
        s, e = token_shard(M, world, r)
        if e > s:
            y[s:e].copy_(gathered[r * per:r * per + (e - s)])
    return y
