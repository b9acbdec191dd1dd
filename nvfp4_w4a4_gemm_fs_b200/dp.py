"""Data-parallel plumbing of the SpliceGEMM path over torch.distributed (NCCL on GPUs, gloo on CPU).

FourSight §5.2 "System Implementation": channel moments are accumulated by a forward hook over the
tokens each rank sees, the protected set is reselected from the moments of the whole step, and the
packed weights (the NVFP4 pack of W with the protected lanes zeroed, and W'_S) are synchronised to
the other engines without requantisation.  With tokens split over ranks:

* ``allreduce_stats``: the one exchange the selection needs.  The moments are exact integers, so
  SUM of n, s1, s2 and MAX of the per-channel maxima (non-negative float bits order as integers)
  and of the range flags give every rank the full batch's state bit for bit, whatever the
  reduction order, and every rank then selects the same channels.
* ``broadcast_packed``: one rank's pre-split (codes, tiled scales, side columns, gains, alpha) sent
  to every rank as raw bytes; receivers skip fs_prepare_weights and hold identical operands.

Collectives only: no kernel here reads another GPU's memory.  Every rank must make the same calls in
the same order.
"""
from __future__ import annotations

import torch
import torch.distributed as dist

__all__ = ["allreduce_stats", "broadcast_packed", "packed_tensors"]


def allreduce_stats(state, group=None) -> None:
    """In-place SUM of the integer moments and row counts, MAX of the per-channel maxima and flags.

    ``state`` is a StatsState (or any object with n, s1, s2, amax, flags tensors of it)."""
    dist.all_reduce(state.s1, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(state.s2, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(state.n, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(state.amax, op=dist.ReduceOp.MAX, group=group)
    dist.all_reduce(state.flags, op=dist.ReduceOp.MAX, group=group)


def packed_tensors(packed, *extra) -> list:
    """The tensors that make up a pre-split weight: codes, tiled scales, side columns (when p > 0),
    then any extra tensors (gains, alpha)."""
    out = [packed.q, packed.sf]
    if packed.p:
        out.append(packed.side)
    out.extend(t for t in extra if t is not None)
    return out


def _broadcast_bytes(t: torch.Tensor, src: int, group) -> None:
    """Broadcast a tensor's bytes (any dtype; a non-contiguous view goes through a contiguous copy)."""
    if t.numel() == 0:
        return
    if t.is_contiguous():
        dist.broadcast(t.view(-1).view(torch.uint8), src=src, group=group)
    else:
        tmp = t.contiguous()
        dist.broadcast(tmp.view(-1).view(torch.uint8), src=src, group=group)
        t.copy_(tmp)


_MAX_PARTS = 8


def _agree_on_sizes(tensors, src: int, group) -> None:
    """Every rank compares its tensor count and byte counts with rank ``src``'s before any data
    moves, and all ranks learn the outcome together (a broadcast of ``src``'s fixed-size header,
    then a MAX all-reduce of the mismatch flag), so a wrong receiver buffer raises on every rank
    instead of leaving ranks in broadcasts of different sizes."""
    if len(tensors) > _MAX_PARTS:
        raise ValueError(f"broadcast_packed: at most {_MAX_PARTS} tensors")
    dev = tensors[0].device
    head = [len(tensors)] + [t.numel() * t.element_size() for t in tensors]
    mine = torch.tensor(head + [0] * (_MAX_PARTS + 1 - len(head)), dtype=torch.int64, device=dev)
    ref = mine.clone()
    dist.broadcast(ref, src=src, group=group)
    bad = torch.tensor([0 if torch.equal(ref, mine) else 1], dtype=torch.int64, device=dev)
    dist.all_reduce(bad, op=dist.ReduceOp.MAX, group=group)
    if int(bad.item()):
        raise ValueError(f"broadcast_packed: buffer sizes differ between ranks (rank {dist.get_rank(group)}: "
                         f"{mine.tolist()}, rank {src}: {ref.tolist()})")


def broadcast_packed(packed, gW=None, alpha=None, src: int = 0, group=None) -> None:
    """Send rank ``src``'s packed weights (q, sf, side) and, when given, its gW and alpha to every
    rank of ``group`` in place.  Receivers must hold buffers of the same shapes (alloc_packed with the
    same N, K, p); their contents are overwritten byte for byte.  The sizes are compared first on
    every rank; a mismatch raises ValueError on all ranks and nothing is sent."""
    tensors = packed_tensors(packed, gW, alpha)
    _agree_on_sizes(tensors, src, group)
    for t in tensors:
        _broadcast_bytes(t, src, group)
