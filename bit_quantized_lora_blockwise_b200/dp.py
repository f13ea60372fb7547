"""Data-parallel exchange step: the sum of the adapter gradients across
ranks (one process per GPU, torch.distributed; NCCL on GPUs, gloo on CPU).

Each rank holds a replica of the quantized frozen weight and runs the layer
on its own tokens; the only data that must cross ranks are the adapter
gradients dA [K, r] and dB [r, N] of every linear, summed in fp32 with one
all-reduce per step (a few MB), then written back in bf16.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def allreduce_adapter_grads(grads, group=None) -> None:
    """In place: every tensor in `grads` becomes its sum over the ranks of
    `group`. All ranks must pass tensors of the same shapes in the same order."""
    if not grads:
        return
    flat = torch.cat([g.reshape(-1).to(torch.float32) for g in grads])
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    off = 0
    for g in grads:
        n = g.numel()
        g.copy_(flat[off:off + n].view_as(g))
        off += n
