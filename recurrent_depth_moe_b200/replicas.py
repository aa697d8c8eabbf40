"""Host-side plumbing of data-parallel replicas (one process per GPU).

The recurrent block shards by sequence with no exchange: causal attention stays inside a
sequence, the MoE has no capacity coupling and ACT is per position.  So N GPUs run N
independent replicas of the block on different sequences; the only collectives are the
timing reductions here (max of the step time, sum of the work done)."""
from __future__ import annotations

import torch
import torch.distributed as dist


def world() -> tuple:
    """(rank, world size) of the default process group, (0, 1) without one."""
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(), dist.get_world_size()
    return 0, 1


def replica_input_seed(seed: int, rank: int) -> int:
    """Each replica draws its own sequences (weights are identical on every rank)."""
    return seed + 101 * rank


def shard_sequences(n_seq: int, rank: int, world_size: int) -> range:
    """Contiguous block of sequence indices owned by `rank` (sizes differ by at most 1)."""
    base, extra = divmod(n_seq, world_size)
    start = rank * base + min(rank, extra)
    return range(start, start + base + (1 if rank < extra else 0))


def max_over_ranks(value: float, device=None) -> float:
    """Step time of the job = the slowest rank's."""
    rank, ws = world()
    if ws == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, device=None) -> float:
    """Work of the job = the sum over ranks."""
    rank, ws = world()
    if ws == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())
