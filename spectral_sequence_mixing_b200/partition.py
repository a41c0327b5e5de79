"""Splitting one causal convolution over several GPUs (one process per GPU).

Every (batch b, channel d) row of r[b, t, d] = sum_{j<=t} v[b, j, d] g[b, t-j, d]
is independent of every other row (Caracal: Causal Architecture via Spectral
Mixing, "Key design 1": the convolution runs per channel; the heads only group
the gate's Conv1d_G2), so the work shards with no exchange step at all:

  * over B in contiguous slabs of batches when there are at least as many
    batches as ranks;
  * otherwise over D in contiguous slabs of channels (a long-context call
    such as [1, 65536, 1024] has one batch).

A rank convolves its own slab with the single-GPU entry points: a batch slab
is already a contiguous [b1-b0, L, D] tensor; a channel slab is made one
([B, L, d1-d0], the layout a tensor-parallel split of the heads gives each GPU
anyway).  Nothing on the data path crosses GPUs; ``gather`` exists only for a
caller that wants all of r on every rank.  This module is host logic only:
slicing and one optional all-gather.
"""
from __future__ import annotations

from dataclasses import dataclass


@dataclass(frozen=True)
class Shard:
    """Rows [b0, b1) x [d0, d1) of a [B, L, D] problem, owned by one rank."""
    axis: str  # "B" or "D": the axis the problem is split along
    b0: int
    b1: int
    d0: int
    d1: int

    @property
    def shape_bd(self):
        return self.b1 - self.b0, self.d1 - self.d0


def _slab(n: int, world: int, rank: int):
    """[lo, hi) of slab `rank` when n items go to `world` ranks as evenly as
    possible (the first n % world slabs one larger)."""
    q, r = divmod(n, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def shard_for(B: int, D: int, world: int, rank: int) -> Shard:
    """The slab of rows rank `rank` of `world` owns: batches when B >= world,
    else channels.  With more ranks than channels some ranks own no rows."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} of world {world}")
    if B < 1 or D < 1:
        raise ValueError(f"B = {B}, D = {D}")
    if B >= world:
        b0, b1 = _slab(B, world, rank)
        return Shard("B", b0, b1, 0, D)
    d0, d1 = _slab(D, world, rank)
    return Shard("D", 0, B, d0, d1)


def take(x, s: Shard):
    """Rank-local slab of a [B, L, D] array (torch tensor or numpy array) as a
    contiguous array: a view for a batch slab, a copy for a channel slab."""
    part = x[s.b0:s.b1, :, s.d0:s.d1]
    if hasattr(part, "contiguous"):
        return part.contiguous()
    import numpy as np
    return np.ascontiguousarray(part)


def place(full, part, s: Shard) -> None:
    """Write a rank's slab of r back into the [B, L, D] array `full`."""
    full[s.b0:s.b1, :, s.d0:s.d1] = part


def gather(part, B: int, L: int, D: int, world: int, rank: int, group=None):
    """All of r on every rank: an all-gather of the ranks' slabs (zero-padded
    to the largest slab, then placed).  Needed only when a caller wants the
    whole result in one place; the convolution itself exchanges nothing."""
    import torch
    import torch.distributed as dist
    shards = [shard_for(B, D, world, q) for q in range(world)]
    nb = max(sh.shape_bd[0] for sh in shards)
    nd = max(sh.shape_bd[1] for sh in shards)
    buf = torch.zeros((nb, L, nd), dtype=part.dtype, device=part.device)
    mine = shards[rank]
    buf[:mine.shape_bd[0], :, :mine.shape_bd[1]] = part
    bufs = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(bufs, buf, group=group)
    full = torch.empty((B, L, D), dtype=part.dtype, device=part.device)
    for sh, b in zip(shards, bufs):
        place(full, b[:sh.shape_bd[0], :, :sh.shape_bd[1]], sh)
    return full
