"""Batch sharding of independent sequences over the ranks of a torch.distributed group.

The sequences of a batch (the breadth workload's samples) are independent problems: each rank
holds a contiguous shard of them, runs the whole path (mining on its shard's pooled prefill,
quantize-append, decode) with no data-path collective, and the decode outputs are gathered once
per step so that every rank holds the output of the whole batch.  Plumbing only: the shards'
arithmetic all runs in libkvq.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_range(num_seqs: int, rank: int, world: int) -> tuple[int, int]:
    """Sequences [b0, b1) of rank `rank`: contiguous, sizes differing by at most one."""
    if world < 1 or not 0 <= rank < world or num_seqs < 0:
        raise ValueError(f"bad shard request: {num_seqs} sequences, rank {rank} of {world}")
    base, extra = divmod(num_seqs, world)
    b0 = rank * base + min(rank, extra)
    return b0, b0 + base + (1 if rank < extra else 0)


def gather_outputs(out_local: torch.Tensor, num_seqs: int, group=None) -> torch.Tensor:
    """All-gather the per-rank decode outputs [b1 - b0, Hq, D] into [num_seqs, Hq, D] on every
    rank (shards padded to the largest one for the collective, then trimmed)."""
    world = dist.get_world_size(group)
    if world == 1:
        return out_local
    sizes = [shard_range(num_seqs, r, world) for r in range(world)]
    most = max(b1 - b0 for b0, b1 in sizes)
    pad = torch.zeros((most,) + tuple(out_local.shape[1:]), dtype=out_local.dtype, device=out_local.device)
    pad[:out_local.shape[0]].copy_(out_local)
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([p[:b1 - b0] for p, (b0, b1) in zip(parts, sizes)], dim=0)
