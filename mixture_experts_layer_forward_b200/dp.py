"""Data-parallel host logic for running the layer on several GPUs.

The MoE layer forward is independent per token (Comet: Fine-grained Computation-
communication Overlapping for Mixture-of-Experts, §2.1: routing, expert FFN and the top-k
reduce all act on one token at a time), so replicas need no data-path collective: every
rank holds the full weights and runs its own batch. The only cross-rank traffic is the
timing reduction (max over ranks) and barriers.
"""
from __future__ import annotations

import os

import torch
import torch.distributed as dist


def env_rank():
    """(rank, local_rank, world_size) from the torchrun environment (defaults 0, 0, 1)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def replica_x_seed(seed: int, rank: int) -> int:
    """Seed of rank r's activations: every replica draws its own batch, weights are shared."""
    return int(seed) * 7919 + 101 * int(rank) + 1


def shard_tokens(T_total: int, rank: int, world: int):
    """Contiguous token shard [start, start + count) of rank `rank` (strong-scaling split)."""
    base, rem = divmod(int(T_total), int(world))
    count = base + (1 if rank < rem else 0)
    start = rank * base + min(rank, rem)
    return start, count


def max_over_ranks(value: float, device=None) -> float:
    """Max of a host scalar across ranks (identity when not distributed)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if dist.is_available() and dist.is_initialized():
        if device is not None and dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
