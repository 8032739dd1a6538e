"""Data-parallel plumbing for the scan: batch sharding and the gradient exchange.

Every (batch, channel) recurrence is independent, so batch rows shard across
ranks with no communication in the forward or the backward of the scan
itself.  The only exchange data-parallel training has is the sum over ranks
of the parameter gradients dA (dim, N), dD (dim,) and ddelta_bias (dim,):
they are packed into one contiguous fp32 buffer so that a single all-reduce
(NCCL on GPUs, gloo on CPU) carries them.
"""
from __future__ import annotations

from typing import Dict, Tuple

import torch
import torch.distributed as dist


def shard_rows(batch: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) batch rows of `rank` (earlier ranks take the remainder)."""
    if world <= 0 or not 0 <= rank < world:
        raise ValueError(f"bad rank {rank} of {world}")
    base, extra = divmod(batch, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def param_grad_buffer(dim: int, dstate: int, device) -> Tuple[torch.Tensor, Dict[str, torch.Tensor]]:
    """One fp32 buffer with views dA (dim, N), dD (dim,), ddelta_bias (dim,)."""
    buf = torch.empty(dim * dstate + 2 * dim, device=device, dtype=torch.float32)
    views = {"dA": buf[:dim * dstate].view(dim, dstate),
             "dD": buf[dim * dstate:dim * dstate + dim],
             "ddelta_bias": buf[dim * dstate + dim:]}
    return buf, views


def allreduce_param_grads(buf: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the packed parameter gradients over the ranks of `group` (in place)."""
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(buf, op=dist.ReduceOp.SUM, group=group)
    return buf
