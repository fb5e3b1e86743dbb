"""Data-parallel plumbing for the QLoRA NF4 linear.

Every rank holds the whole 4-bit weight and processes its own tokens.  Y and
dX are per token and need no exchange; dA = dH^T X and dB = s dY^T H are sums
over tokens, so each rank's partial gradients are summed across ranks (the
one collective of the path, NCCL on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def token_shard(M_total: int, rank: int, world: int) -> tuple[int, int]:
    """[start, end) of this rank's tokens: contiguous, sizes differ by at most one."""
    base, extra = divmod(M_total, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None, average: bool = False) -> None:
    """Sums dA and dB over the ranks of `group` in place (optionally averaged)."""
    dist.all_reduce(dA, group=group)
    dist.all_reduce(dB, group=group)
    if average:
        w = dist.get_world_size(group)
        dA.div_(w)
        dB.div_(w)
