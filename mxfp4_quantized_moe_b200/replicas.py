"""Data-parallel replicas of the expert block (one process per GPU).

The layer has no weight gradient and maps every token independently, so N GPUs run N
independent batches of tokens against replicated weights: no collective touches the data
path.  The only cross-rank steps are host-side bookkeeping for measurement:

* each rank draws its own batch (seed offset by rank) while the weights are shared;
* the step time is the maximum over ranks, and the throughput counts every rank's tokens.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

RANK_SEED_STRIDE = 1000


def batch_seed(seed: int, rank: int) -> int:
    """Seed of a rank's token batch (rank 0 keeps the base seed, so N=1 matches the workload)."""
    return seed + RANK_SEED_STRIDE * rank


def max_over_ranks(value: float, device=None) -> float:
    """Largest `value` over all ranks (identity without an initialized process group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(tokens_per_rank: int, steps: int, max_ms: float, world: int) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's time."""
    return tokens_per_rank * world * steps / (max_ms / 1e3)
