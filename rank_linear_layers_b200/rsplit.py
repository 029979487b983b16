"""Tensor parallelism over the inner rank r of Y = (X·A)·B (+bias).

Splitting r across the ranks of a process group makes each rank's work a
smaller low-rank layer: rank i holds A[:, r_i0:r_i1] and B[r_i0:r_i1, :],
computes its partial product P_i = (X·A_i)·B_i in fp32 with the library's
kernels, and one all-reduce (NCCL over NVLink) sums the partials:
Y = Σ_i P_i (+bias, added on one rank only).  The slices start on multiples
of 16, so each rank's factors keep 32-byte-aligned rows when the whole rank
does (the GAC paper's point, §3, that a dimension's alignment sets its
speed, applies to every piece of a split).

The all-reduce is torch.distributed's (the library's kernels compute; NCCL
moves the partial sums).  Nothing here runs the reduction or the product on
the CPU: `local_product` exists so that the split and the reduction can be
checked on CPU ranks with a reference product.
"""
from __future__ import annotations

from typing import Callable, Optional, Tuple


def rsplit_bounds(r: int, world: int, rank: int, align: int = 16) -> Tuple[int, int]:
    """Rank `rank`'s slice [r0, r1) of the inner dimension r split over
    `world` ranks: slices start on multiples of `align` and are as even as
    that allows (the last may be shorter; trailing ranks may be empty when
    r < world·align)."""
    if r < 0 or world < 1 or not 0 <= rank < world or align < 1:
        raise ValueError("bad split")
    units = -(-r // align)                      # align-sized pieces of r
    u0 = units * rank // world
    u1 = units * (rank + 1) // world
    return min(r, u0 * align), min(r, u1 * align)


def _library_partial(X, A_part, B_part, bias):
    from . import lr_linear_f32
    return lr_linear_f32(X, A_part, B_part, bias)


def lr_linear_rsplit(X, A_part, B_part, bias=None, group=None,
                     local_product: Optional[Callable] = None):
    """fp32 Y = (X·A)·B (+bias) with r split over the ranks of `group`.

    X [M, K] (every rank), A_part [K, r_i], B_part [r_i, N] (this rank's
    slice, see rsplit_bounds), bias [N] or None (used by group rank 0 only).
    Returns the fp32 [M, N] sum on every rank (one all-reduce)."""
    import torch.distributed as dist
    rank = dist.get_rank(group) if dist.is_initialized() else 0
    world = dist.get_world_size(group) if dist.is_initialized() else 1
    product = local_product or _library_partial
    P = product(X, A_part, B_part, bias if rank == 0 else None)
    if world > 1:
        dist.all_reduce(P, op=dist.ReduceOp.SUM, group=group)
    return P
