"""Host-side plumbing of data-parallel replicas (one process per GPU).

The layer shards by tokens with no exchange: every GPU holds all experts and
runs the whole forward on its own batch, so N GPUs are N independent
replicas (capacity, keep-fraction and expert choice then act per shard, as
GShard's local groups do).  Nothing here touches the data path; it covers
rank discovery, per-rank input seeds, and the max-over-ranks timing the
benchmark reports.  torch.distributed is used only for a barrier and one
all-reduce of a scalar.
"""
from __future__ import annotations

import os
from dataclasses import dataclass


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info(env=os.environ) -> RankInfo:
    """Rank, world size and local rank from the torchrun environment (1 GPU if unset)."""
    return RankInfo(int(env.get("RANK", "0")), int(env.get("WORLD_SIZE", "1")),
                    int(env.get("LOCAL_RANK", "0")))


def token_seed(seed: int, rank: int, world: int) -> int:
    """Seed of a rank's token batch.  One GPU keeps the plain seed; with N > 1
    every rank draws its own tokens.  Weights always use the plain seed, so
    every replica holds the same layer."""
    return seed if world == 1 else seed * 1000 + rank + 1


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The largest `value` over all ranks (the value itself without a group)."""
    if dist is None or not dist.is_initialized():
        return float(value)
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world: int, tokens_per_rank: int, steps: int, max_total_ms: float) -> float:
    """Whole-job tokens/s: tokens of all ranks over the slowest rank's time."""
    return world * tokens_per_rank * steps / (max_total_ms / 1e3)
