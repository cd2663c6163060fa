"""Tensor-parallel partitions of a packed weight (host-side slicing only).

The packed planes are row-major ([N][K/32] index words and sign bytes, scales
[N][K/group], [N] or [1]), so the method's data parallelism maps onto two
partitions without re-quantisation:

* N-split (column-parallel): rank r keeps output rows [r0, r1) -- their index
  words, sign bytes and group or row scales, unchanged (a per-tensor scale is
  copied to every rank).  Each rank computes Y[:, r0:r1]; an all-gather of the
  shards along N gives Y.
* K-split (row-parallel): rank r keeps the weights of K range [k0, k1), cut at
  scale-group boundaries (whole packed words, whole groups), and the matching
  slice of X.  Each rank computes a partial Y over its K range; an all-reduce
  (sum) of the partials gives Y, equal to the unsplit result within the fp32
  summation-order bound.  Row and tensor scales apply to every K range alike.

These functions only slice torch tensors; the linear itself runs through the
library on each rank's GPU, and the exchange is a torch.distributed (NCCL over
NVLink) collective.  Quantising a weight across ranks with per-channel or
per-tensor scales would need the canonical pairwise sums gathered in tree
order; quantisation is done before sharding here.
"""
from __future__ import annotations

from . import PER_CHANNEL, PER_GROUP, PER_TENSOR, PackedWeight


def bounds(n: int, world: int, rank: int, align: int = 1) -> tuple[int, int]:
    """[lo, hi) of an even split of range(n) into `world` parts whose inner
    boundaries are multiples of `align` (the last part takes the remainder)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank or world size")
    units = n // align
    base, extra = divmod(units, world)
    lo = align * (rank * base + min(rank, extra))
    hi = align * ((rank + 1) * base + min(rank + 1, extra))
    if rank == world - 1:
        hi = n
    return lo, hi


def shard_rows(P: PackedWeight, world: int, rank: int, align: int = 1) -> tuple[PackedWeight, int, int]:
    """N-split: (the rank's packed rows as views, r0, r1)."""
    r0, r1 = bounds(P.N, world, rank, align)
    if P.granularity == PER_TENSOR:
        sc = P.scales
    else:
        spr = 1 if P.granularity == PER_CHANNEL else P.K // P.group
        sc = P.scales[r0 * spr:r1 * spr]
    return PackedWeight(P.idx[r0:r1], P.sgn[r0:r1], sc, r1 - r0, P.K, P.granularity, P.group), r0, r1


def shard_k(P: PackedWeight, world: int, rank: int) -> tuple[PackedWeight, int, int]:
    """K-split at scale-group boundaries (whole packed words for row scales):
    (the rank's packed columns, copied contiguous, k0, k1)."""
    step = P.group if P.granularity == PER_GROUP else 32
    if P.granularity == PER_GROUP and P.group % 32:
        raise ValueError("group must be a multiple of 32")
    k0, k1 = bounds(P.K, world, rank, step)
    w0, w1 = k0 // 32, k1 // 32
    idx = P.idx[:, w0:w1].contiguous()
    sgn = P.sgn[:, w0:w1].contiguous()
    if P.granularity == PER_GROUP:
        g = P.K // P.group
        sc = P.scales.view(P.N, g)[:, k0 // P.group:k1 // P.group].contiguous().view(-1)
    else:
        sc = P.scales
    return PackedWeight(idx, sgn, sc, P.N, k1 - k0, P.granularity, P.group), k0, k1


def gather_rows(y_shard, world: int, group=None):
    """All-gather of N-split shards [M, n_r] into Y [M, N] (equal shard widths:
    N divisible by world; torch.distributed must be initialised)."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(y_shard) for _ in range(world)]
    dist.all_gather(parts, y_shard.contiguous(), group=group)
    return torch.cat(parts, dim=1)


def reduce_k(y_partial, group=None):
    """All-reduce (sum) of K-split partial outputs, in place."""
    import torch.distributed as dist
    dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
    return y_partial
