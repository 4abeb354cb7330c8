"""One process per GPU for the decode path.

Decode of one sequence reads nothing of another, so the path partitions by
sequence: every rank decodes its own batch and no collective touches the
data path.  The only cross-rank traffic is in measurement: a barrier around
the timed region and one all-reduce (MAX) of the elapsed device time.

The path also partitions by group within one batch (tensor parallelism over
heads, "GQLA" scholarbro.com Abstract: the GQA path shards its per-group
cache over up to 8 GPUs with no redundancy, while the absorb path keeps the
whole latent cache on every rank).  A group's heads attend only to that
group's K/V, so a rank holding groups [g0, g1) and their heads computes those
heads' outputs alone; the exchange comes after the output projection, outside
this path.  `tp_shard` cuts one rank's share out of a batch.
"""
from __future__ import annotations

import dataclasses
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


def tp_groups(G: int, world: int, rank: int):
    """Groups [g0, g1) of `rank` when G groups are split evenly over `world` ranks."""
    if world < 1 or not 0 <= rank < world or G % world != 0:
        raise ValueError("G = %d groups do not split evenly over %d ranks" % (G, world))
    per = G // world
    return rank * per, (rank + 1) * per


def tp_shard(inp, world: int, rank: int):
    """This rank's share of a batch under group tensor parallelism: its groups'
    heads of q, its groups' up-projections, the dims of a layer with n_h/world
    heads and G/world groups.  The latent cache, lengths and block table are
    the same tensors on every rank (the absorb path reads all of it; the GQA
    path expands only its own groups from it)."""
    d = inp.dims
    g0, g1 = tp_groups(d.G, world, rank)
    m = d.n_h // d.G
    dims = dataclasses.replace(d, n_h=d.n_h // world, G=d.G // world, scale=d.softmax_scale)
    wl = dataclasses.replace(inp.wl, dims=dims)
    return dataclasses.replace(inp, wl=wl, q=inp.q[:, :, g0 * m:g1 * m].contiguous(),
                               W_uk=inp.W_uk[g0:g1].contiguous(), W_uv=inp.W_uv[g0:g1].contiguous())
