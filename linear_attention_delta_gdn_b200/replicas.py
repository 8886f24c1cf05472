"""Host-side logic of running the operator as independent replicas, one process per GPU.

(batch, head) pairs never interact, so N ranks each process their own batch with no
data-path collective (weak scaling). The process group is used only to align the timed
region (barrier) and to take the slowest rank's time.
"""
from __future__ import annotations

RANK_SEED_STRIDE = 7919


def rank_seed(seed: int, rank: int) -> int:
    """Seed of rank `rank`'s synthetic batch (rank 0 draws the workload's own inputs)."""
    return seed + RANK_SEED_STRIDE * rank


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Largest `value` over all ranks (identity without an initialised process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tokens_per_s(world: int, tokens_per_rank_step: int, ms_per_step_slowest: float) -> float:
    """Whole-job throughput: all ranks' tokens of one step over the slowest rank's step time."""
    return world * tokens_per_rank_step / (ms_per_step_slowest / 1e3)
