"""Splitting one packed image batch across GPUs.

Attention never crosses images, so the images of a cu_seqlens-packed batch
can be divided among ranks with no exchange on the attention path.  The one
exchange is the dynamic per-tensor scale: every rank must quantize with the
descales of the whole batch, so the three amax values (q, k, v) are
all-reduced with max before the ring update (fp8_amax3 -> all-reduce ->
fp8_ring_push).  Host logic only; the device work stays in the kernels.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shard_images(seg_lens, world_size: int, rank: int) -> list[int]:
    """Indices of the images rank `rank` takes: longest-processing-time-first
    assignment on the attention cost S^2 (ties by lower index), deterministic
    on every rank."""
    if world_size < 1 or not 0 <= rank < world_size:
        raise ValueError("bad world_size / rank")
    order = sorted(range(len(seg_lens)), key=lambda i: (-int(seg_lens[i]) ** 2, i))
    load = [0] * world_size
    owner = [0] * len(seg_lens)
    for i in order:
        r = min(range(world_size), key=lambda w: (load[w], w))
        owner[i] = r
        load[r] += int(seg_lens[i]) ** 2
    return [i for i in range(len(seg_lens)) if owner[i] == rank]


def local_batch(seg_lens, world_size: int, rank: int):
    """(image indices, local segment lengths, [(start, end) token ranges of
    those images in the global packing])."""
    starts = [0]
    for s in seg_lens:
        starts.append(starts[-1] + int(s))
    ids = shard_images(seg_lens, world_size, rank)
    return ids, [int(seg_lens[i]) for i in ids], [(starts[i], starts[i + 1]) for i in ids]


def allreduce_amax3(amax3: torch.Tensor, group=None) -> torch.Tensor:
    """In-place all-reduce(max) of the three per-tensor amax values."""
    dist.all_reduce(amax3, op=dist.ReduceOp.MAX, group=group)
    return amax3
