"""Data parallelism over tokens for the LoRA linear layer.

Each rank processes its own tokens with its own copy of the frozen weight and the
adapter; the only quantities that must be combined are the adapter gradients,
dA = s·Σ_m (dY·B)[m]ᵀ X[m] and dB = s·Σ_m dY[m]ᵀ XA[m], which are sums over tokens and
therefore sums over ranks.  Y and dX stay local to the rank that owns the tokens.  The
data-parallel wrapper with a custom all-reduce is the distributed-training paragraph of
"Unsloth vs The Stack v2"; it names no precision for the exchange.  Here the ranks' fp32
partial sums are exchanged and the total is rounded to bf16 once
(:class:`AdapterGradExchange`), so the result does not depend on the number of ranks
beyond fp32 summation order.
"""
from __future__ import annotations

import math

import torch
import torch.distributed as dist


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """Sum dA and dB over the ranks of `group` in place, in their own dtype (NCCL on
    GPUs, gloo on CPUs).  For bf16 gradients this rounds twice (each rank's value, then
    every partial sum); :class:`AdapterGradExchange` exchanges fp32 instead."""
    if not dist.is_initialized() or dist.get_world_size(group) == 1:
        return
    dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group)


def _library_round(src: torch.Tensor, dst: torch.Tensor) -> None:
    from .binding import lora_round_bf16
    lora_round_bf16(src, dst)


class AdapterGradExchange:
    """fp32 adapter gradients of one data-parallel step in one flat buffer.

    ``views`` are fp32 tensors of the given shapes inside one buffer (each starting on a
    16-byte boundary); the backward writes the unrounded gradients into them
    (``LORA_GRADS_F32``), :meth:`allreduce` sums the whole buffer over the ranks with one
    collective, and :meth:`round_into` writes each sum, rounded to nearest even once, into
    the caller's bf16 tensors (with the library's kernel unless ``round_fn`` is given)."""

    def __init__(self, shapes, device, round_fn=None):
        self.shapes = [tuple(int(d) for d in s) for s in shapes]
        sizes = [math.prod(s) for s in self.shapes]
        offs, off = [], 0
        for n in sizes:
            offs.append(off)
            off += (n + 3) // 4 * 4  # 16-byte aligned starts
        self.flat = torch.zeros(max(off, 1), dtype=torch.float32, device=device)
        self.views = [self.flat[o:o + n].view(s) for o, n, s in zip(offs, sizes, self.shapes)]
        self.round_fn = round_fn or _library_round

    @property
    def nbytes(self) -> int:
        return self.flat.numel() * 4

    def allreduce(self, group=None) -> None:
        if dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)

    def round_into(self, outs) -> None:
        if len(outs) != len(self.views):
            raise ValueError("one output per gradient")
        for v, o in zip(self.views, outs):
            if tuple(o.shape) != tuple(v.shape) or o.dtype != torch.bfloat16:
                raise ValueError(f"output {tuple(o.shape)} {o.dtype} for a gradient of shape {tuple(v.shape)}")
            self.round_fn(v, o)


def token_shard(M_total: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous token range [start, stop) of `rank` when M_total tokens are split over
    `world` ranks (the first M_total % world ranks take one extra token)."""
    base, extra = divmod(M_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)
