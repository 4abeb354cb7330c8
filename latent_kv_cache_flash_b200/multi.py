"""One process per GPU for the decode path.

Decode of one sequence reads nothing of another, so the path partitions by
sequence: every rank decodes its own batch and no collective touches the
data path.  The only cross-rank traffic is in measurement: a barrier around
the timed region and one all-reduce (MAX) of the elapsed device time.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def rank_info():
    """(rank, local_rank, world_size) from the torchrun environment."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def rank_seed(base_seed: int, rank: int) -> int:
    """Each rank draws an independent batch."""
    return base_seed + rank


def barrier():
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device="cpu") -> float:
    """The slowest rank's time: the job finishes when the last rank does."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: tokens decoded by all ranks / the max-over-ranks time."""
    return world * tokens_per_rank_step * steps / (max_ms * 1e-3)
