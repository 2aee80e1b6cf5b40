"""Data parallelism for the streamed LoRA step.

One process per GPU: every rank streams its own copy of the frozen base over
its own host link and runs its own micro-batch through the whole step; the
LoRA gradients, the only trained state, are averaged across ranks once per
step.  They live in one flat fp32 buffer (each factor a view into it that
starts on a 512-byte boundary, 256 bytes for the bf16 working copies laid out
the same way), so the exchange is a single in-place all-reduce of that buffer;
the 1/world of the mean can be left to the optimiser step (its gradient
scale), which reads the buffer anyway.
"""
from __future__ import annotations

import torch

ALIGN = 128  # elements (512 bytes of fp32, 256 of bf16)


def flat_layout(shapes):
    """Offsets (in elements) of tensors of the given shapes packed in order,
    each starting on a multiple of ALIGN elements, and the total length."""
    offs, n = [], 0
    for sh in shapes:
        offs.append(n)
        size = 1
        for d in sh:
            size *= int(d)
        n += (size + ALIGN - 1) // ALIGN * ALIGN
    return offs, n


def flat_views(shapes, device, dtype=torch.float32):
    """A zeroed flat buffer and one contiguous view per shape (see flat_layout)."""
    offs, n = flat_layout(shapes)
    flat = torch.zeros(max(n, 1), dtype=dtype, device=device)
    views = []
    for o, sh in zip(offs, shapes):
        size = 1
        for d in sh:
            size *= int(d)
        views.append(flat[o:o + size].view(sh))
    return flat, views


def allreduce_mean_(flat: torch.Tensor, group=None) -> torch.Tensor:
    """Average `flat` over the process group in place: one all-reduce (sum)
    and one scale by 1/world.  A no-op when torch.distributed is not
    initialised or the group has a single rank."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return flat
    world = dist.get_world_size(group)
    if world > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
        flat.mul_(1.0 / world)
    return flat


def allreduce_sum_(flat: torch.Tensor, group=None) -> int:
    """Sum `flat` over the process group in place (one all-reduce) and return
    the group's size, so that the caller can fold the 1/world of the mean into
    its next pass over the buffer.  Returns 1 without touching `flat` when
    torch.distributed is not initialised or the group has a single rank."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1
    world = dist.get_world_size(group)
    if world > 1:
        dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    return world
