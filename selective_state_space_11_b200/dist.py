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


# ------------------------------------------------------------ sequence sharding
# For B*D-starved long contexts the sequence itself shards: rank r holds the
# contiguous segment r of L (every batch row and channel).  A segment run from
# an initial state h0 ends in h_end = P o h0 + E (E: its end state from zero,
# P = exp(A sum Delta): the segment's diagonal state transition), so one
# exchange of (P, E) lets every rank rebuild the state entering its segment
# ("mamba-metal" README, "Long-context prompts (parallel prefill)", with the
# pieces on different GPUs).  The backward chains the adjoints the same way in
# reverse and sums the parameter gradients over the ranks.

def shard_seq(seqlen: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [start, stop) steps of `rank` (earlier ranks take the remainder)."""
    return shard_rows(seqlen, rank, world)


class ScanKernels:
    """The library's kernels for the segment steps of sequence sharding.

    A segment is a dict with u, delta, A, B, C, D, z, delta_bias and
    delta_softplus, every sequence-indexed tensor cut to the segment."""

    def fwd(self, seg, h0):
        from . import ops
        return ops.ss_fwd(seg["u"], seg["delta"], seg["A"], seg["B"], seg["C"], D=seg["D"], z=seg["z"],
                          delta_bias=seg["delta_bias"], delta_softplus=seg["delta_softplus"], h0=h0)

    def bwd(self, seg, dy, checkpoints, h0, dfinal):
        from . import ops
        return ops.ss_bwd(seg["u"], seg["delta"], seg["A"], seg["B"], seg["C"], dy, checkpoints, D=seg["D"],
                          z=seg["z"], delta_bias=seg["delta_bias"], delta_softplus=seg["delta_softplus"],
                          h0=h0, dfinal=dfinal, want_dh0=True)

    def decay(self, seg):
        from . import ops
        return ops.segment_decay(seg["delta"], seg["A"], seg["delta_bias"], seg["delta_softplus"])

    def chain(self, P, E, reverse):
        from . import ops
        return ops.state_chain(P, E, None, reverse=reverse)


def all_gather_stacked(t: torch.Tensor, group=None) -> torch.Tensor:
    """(world, *t.shape): every rank's `t`, in rank order (NCCL or gloo)."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(t) for _ in range(world)]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def seq_sharded_forward(seg, h0, rank: int, world: int, gather, kernels=None):
    """Forward of this rank's segment with the true entering state.

    gather(t) -> (world, *t.shape) stacks every rank's t.  Returns (y,
    end_state, checkpoints, h_in, P): y and the checkpoints of this segment,
    its end state (the sequence's final state on the last rank), the state
    that entered it and its transition P (both reused by the backward)."""
    k = kernels or ScanKernels()
    # pass 1: rank 0 from the true h0, the others from zero
    y, end, ck = k.fwd(seg, h0 if rank == 0 else None)
    P = k.decay(seg)
    H = k.chain(gather(P), gather(end), reverse=False)  # H[r]: the state entering segment r, r >= 1
    if rank == 0:
        return y, end, ck, h0, P
    h_in = H[rank].contiguous()
    y, end, ck = k.fwd(seg, h_in)  # pass 2 from the true entering state
    return y, end, ck, h_in, P


def seq_sharded_backward(seg, dy, checkpoints, h_in, P, dfinal, rank: int, world: int, gather, allreduce,
                         kernels=None):
    """Backward of this rank's segment for <dy, y> + <dfinal, final state>.

    `checkpoints`, `h_in` and `P` come from seq_sharded_forward.  allreduce(t)
    sums t over the ranks in place.  Returns the gradient dict of ss_bwd with
    dA, dD, ddelta_bias summed over all segments and, on rank 0, the dh0 of
    the whole sequence."""
    k = kernels or ScanKernels()
    last = world - 1
    # pass 1: the last rank with the true dfinal, the others with a zero adjoint at their end
    g = k.bwd(seg, dy, checkpoints, h_in, dfinal if rank == last else None)
    G = k.chain(gather(P), gather(g["dh0"]), reverse=True)  # G[r]: the adjoint reaching the end of segment r
    if rank < last:
        g = k.bwd(seg, dy, checkpoints, h_in, G[rank].contiguous())  # pass 2
    dim, N = g["dA"].shape
    buf = torch.cat([g["dA"].reshape(-1), g["dD"].reshape(-1) if g.get("dD") is not None else
                     torch.zeros(dim, dtype=g["dA"].dtype, device=g["dA"].device),
                     g["ddelta_bias"].reshape(-1) if g.get("ddelta_bias") is not None else
                     torch.zeros(dim, dtype=g["dA"].dtype, device=g["dA"].device)])
    allreduce(buf)
    g = dict(g)
    g["dA"] = buf[:dim * N].view(dim, N)
    g["dD"] = buf[dim * N:dim * N + dim]
    g["ddelta_bias"] = buf[dim * N + dim:]
    return g
