"""Data parallelism over tokens for the LoRA linear layer.

Each rank processes its own tokens with its own copy of the frozen weight and the
adapter; the only quantities that must be combined are the adapter gradients,
dA = s·Σ_m (dY·B)[m]ᵀ X[m] and dB = s·Σ_m dY[m]ᵀ XA[m], which are sums over tokens and
therefore sums over ranks.  Y and dX stay local to the rank that owns the tokens.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """Sum dA and dB over the ranks of `group` in place (NCCL on GPUs, gloo on CPUs)."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group)


def token_shard(M_total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous token range [start, stop) of `rank` when M_total tokens are split over
    `world` ranks (the first M_total % world ranks take one extra token)."""
    base, extra = divmod(M_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)
