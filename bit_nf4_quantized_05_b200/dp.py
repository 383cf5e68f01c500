"""Data-parallel plumbing for the QLoRA layer (one process per GPU).

The frozen NF4 weight and the adapters are replicated; every rank runs the
layer's forward and backward on its own tokens, so the forward needs no
communication. The only exchange is the adapter-gradient reduction: dA and dB
live in one flat buffer per rank and are averaged with a single all-reduce
(NCCL over NVLink on GPUs; gloo in the CPU tests).
"""
from __future__ import annotations

from typing import Tuple

import torch
import torch.distributed as dist


def shard_rows(M: int, rank: int, world: int) -> Tuple[int, int]:
    """[start, stop) of this rank's tokens when M tokens are split as evenly as
    possible (the first M % world ranks take one extra token)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError("bad rank/world")
    base, extra = divmod(M, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def grad_buffer(r: int, k: int, n: int, dtype=torch.float32, device=None):
    """One flat buffer holding dA [r, k] then dB [n, r]; returns (flat, dA, dB).

    fp32 by default: the backward then writes the adapter gradients in fp32
    (qlora_linear_bwd_f32grad) and the ranks sum them in fp32, so the reduced
    gradient carries no bf16 rounding of the per-rank partial sums."""
    flat = torch.empty(r * k + n * r, dtype=dtype, device=device)
    return flat, flat[: r * k].view(r, k), flat[r * k:].view(n, r)


def allreduce_adapter_grads(flat: torch.Tensor, world: int, group=None,
                            average: bool = True) -> torch.Tensor:
    """Sum (or average) the flat adapter-gradient buffer over all ranks, in place.

    Averaging divides by `world` after the sum, so ranks that processed equal
    token counts produce the gradient of the mean loss over all tokens."""
    if world > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        if average:
            flat.div_(world)
    return flat
