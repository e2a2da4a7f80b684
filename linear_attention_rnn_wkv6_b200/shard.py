"""Splitting one WKV problem over GPUs along the batch (one process per GPU).

Every (b, h) unit of the RWKV-6 operator (every (b, c) of RWKV-4) is an
independent problem: each head carries its own state ("RWKV Architecture ...",
Complexity and Operational Scaling; one independent block per (b, h) in "How
Custom CUDA Kernels (wkv6_cuda.cu) ...", Kernel Architecture and Launch
Configuration).  So a batch can be split over ranks with no communication for
the forward; the backward's du, a sum over the batch, is the one exchange: one
all-reduce of C floats over the ranks' partial sums.

This module holds only that plumbing (which batches a rank owns, and the
collective); every step of the operator itself runs in libwkv.so's kernels.
"""
from __future__ import annotations


def batch_range(B: int, rank: int, world: int) -> tuple[int, int]:
    """The contiguous batches [lo, hi) of a B-batch problem that `rank` of `world` owns.

    The ranges of ranks 0..world-1 cover 0..B-1 exactly once, in order, and differ in
    size by at most one batch (the first B % world ranks take one more)."""
    if world < 1 or not 0 <= rank < world or B < 0:
        raise ValueError(f"bad split: B={B} rank={rank} world={world}")
    base, extra = divmod(B, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def allreduce_du(du, group=None) -> None:
    """Sum each rank's du partial (the gradient of u over the rank's batches, a [C]
    tensor) over all ranks, in place: afterwards every rank holds du of the whole
    batch.  One collective of C floats (NCCL over NVLink for CUDA tensors)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(du, op=dist.ReduceOp.SUM, group=group)
