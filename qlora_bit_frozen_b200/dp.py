"""Data-parallel plumbing for the QLoRA linear layer.

The layer shards along tokens: every rank holds a replica of the packed
frozen weight and of the fp32 adapters and runs forward/backward on its own
tokens.  Y and dX stay per rank; the only exchange is the sum of the adapter
gradients dA and dB over ranks (dA = s V^T X and dB = s dY^T U are sums over
tokens, so the sum of per-shard gradients is the full-batch gradient).
torch.distributed carries it (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import Iterable

import torch
import torch.distributed as dist


def allreduce_adapter_grads(grads: Iterable[torch.Tensor], group=None) -> None:
    """Sum each gradient tensor in place over all ranks of `group`, in order.
    Every rank must pass the same sequence of shapes."""
    if not dist.is_available() or not dist.is_initialized():
        return
    if dist.get_world_size(group) == 1:
        return
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)


def allreduce_flat(grads: torch.Tensor, group=None) -> None:
    """Sum one flat gradient arena (every dA and dB of the model laid out
    back to back) in place over all ranks: one collective per step instead
    of one per tensor."""
    if not dist.is_available() or not dist.is_initialized():
        return
    if dist.get_world_size(group) == 1:
        return
    dist.all_reduce(grads, op=dist.ReduceOp.SUM, group=group)


def max_over_ranks(value: float, device="cpu", group=None) -> float:
    """The maximum of a per-rank scalar (step time) over all ranks."""
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def shard_rows(R_total: int, world: int, rank: int):
    """[lo, hi) token range of `rank` when R_total tokens are split over
    `world` ranks as evenly as possible."""
    base, rem = divmod(R_total, world)
    lo = rank * base + min(rank, rem)
    hi = lo + base + (1 if rank < rem else 0)
    return lo, hi
