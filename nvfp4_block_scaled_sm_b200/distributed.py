"""Multi-GPU use of the quantizers, one process per GPU.

MXFP8 needs no exchange: rows (and experts) are independent, so each rank
quantizes its own rows and the results concatenate.

NVFP4 on a tensor sharded along rows has one real exchange: the global
scale g = A / 2688 needs the amax A of the whole tensor ("Add FP8, NVFP4,
and QARL training and export", review: two-level global + block scaling).
Each rank reduces its shard on the GPU (nvfp4_amax), the ranks all-reduce
that single fp32 with MAX (NCCL over NVLink; any torch.distributed backend
works), and each rank then quantizes its shard with the global amax; the
kernel derives g from it, so every rank uses bit-identical scales.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_amax_(amax: torch.Tensor, group=None) -> torch.Tensor:
    """In-place MAX all-reduce of a one-element fp32 amax over `group`."""
    if amax.numel() != 1 or amax.dtype != torch.float32:
        raise TypeError("amax must be a single fp32 value")
    dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def nvfp4_quantize_sharded(x_local: torch.Tensor, group=None):
    """NVFP4 quantize of this rank's row shard with the global scale of the
    whole sharded tensor. Returns (packed, block_scale, global_scale) for
    the local rows; global_scale is identical on every rank."""
    from . import nvfp4_amax, nvfp4_quantize
    amax = nvfp4_amax(x_local)
    allreduce_amax_(amax, group)
    return nvfp4_quantize(x_local, amax=amax)


def shard_rows(M: int, world: int, rank: int) -> tuple[int, int]:
    """[begin, end) of rank's contiguous share of M rows (sizes differ by at
    most one)."""
    base, extra = divmod(M, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)
