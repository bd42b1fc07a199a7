"""Data-parallel sharding of the GSPN propagation across ranks (one process per GPU).

Output planes (n, c) are independent: the forward of a plane depends only on its own x, lambda,
u and the logits of its (n, c) (per-channel) or (n) (channel-shared). So the work is split into
plane shards with no collective on the forward path:

  - batch sharding: rank r takes a contiguous block of the batch axis N (every weight mode);
  - channel sharding (when N is smaller than the number of ranks, e.g. one image with 1152
    channels): rank r takes a contiguous block of channels for every n.

The backward needs one collective only in the channel-shared mode with channel sharding: the
logit gradient of a shared w_i is the sum over channels, so each rank's partial da is summed
across ranks (one all-reduce of D x N x 1 x 3 x H x W values). With batch sharding every rank
owns its batch items' da outright.

This module only computes index ranges and calls torch.distributed; every arithmetic step of the
propagation runs in libgspn on the local shard.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Shard:
    axis: str          # "N" or "C"
    start: int
    stop: int

    @property
    def size(self) -> int:
        return self.stop - self.start


def _block(total: int, parts: int, index: int):
    base, extra = divmod(total, parts)
    start = index * base + min(index, extra)
    return start, start + base + (1 if index < extra else 0)


def plan(N: int, C: int, world: int, rank: int) -> Shard:
    """Contiguous plane shard of `rank`: batch blocks when N >= world, else channel blocks."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad world/rank")
    if N >= world:
        s, e = _block(N, world, rank)
        return Shard("N", s, e)
    if C < world:
        raise ValueError(f"cannot give each of {world} ranks a plane shard of N={N}, C={C}")
    s, e = _block(C, world, rank)
    return Shard("C", s, e)


def take(t: torch.Tensor, shard: Shard, logits: bool = False, shared: bool = False) -> torch.Tensor:
    """The shard's slice of an N x C x H x W tensor, or of D x N x Cw x 3 x H x W logits."""
    if logits:
        if shard.axis == "N":
            return t[:, shard.start:shard.stop]
        return t if shared else t[:, :, shard.start:shard.stop]
    if shard.axis == "N":
        return t[shard.start:shard.stop]
    return t[:, shard.start:shard.stop]


def needs_da_allreduce(shard: Shard, shared: bool) -> bool:
    return shared and shard.axis == "C"


def allreduce_da(da: torch.Tensor, shard: Shard, shared: bool, group=None) -> torch.Tensor:
    """Sums the channel-shared logit gradient across channel shards (in place). Every rank must
    call this at the same point, with the same shape, even when it is a no-op for the plan."""
    if needs_da_allreduce(shard, shared) and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(da, op=dist.ReduceOp.SUM, group=group)
    return da


def forward_shard(x, a, lam, u, wmode: int, dir_mask: int, shard: Shard, **kw):
    """libgspn forward on this rank's shard (contiguous copies of the slices)."""
    from . import forward
    shared = wmode == 1
    xs, ls, us = (take(t, shard).contiguous() for t in (x, lam, u))
    as_ = take(a, shard, logits=True, shared=shared).contiguous()
    return forward(xs, as_, ls, us, wmode, dir_mask, **kw)


def backward_shard(x, a, lam, u, dy, wmode: int, dir_mask: int, shard: Shard, group=None, **kw):
    """libgspn backward on this rank's shard; da is all-reduced when the plan needs it."""
    from . import backward
    shared = wmode == 1
    xs, ls, us, dys = (take(t, shard).contiguous() for t in (x, lam, u, dy))
    as_ = take(a, shard, logits=True, shared=shared).contiguous()
    dx, da, dlam, du = backward(xs, as_, ls, us, dys, wmode, dir_mask, **kw)
    allreduce_da(da, shard, shared, group)
    return dx, da, dlam, du
