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


def token_shard(tokens: int, rank: int, world: int) -> tuple[int, int]:
    """[t0, t1): the contiguous tokens of `rank` when `tokens` are split over
    `world` ranks as evenly as possible (data parallel over M)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    return tokens * rank // world, tokens * (rank + 1) // world


def codec_shard_rows(N: int, K: int, rank: int, world: int) -> tuple[int, int]:
    """[r0, r1): the weight rows `rank` quantizes (or dequantizes) when the
    codec of an [N, K] weight is split over `world` ranks in whole
    second-level groups (256 constants = 16384 consecutive elements of the
    row-major weight), so that no group, and no 64-block, straddles two
    ranks and no exchange is needed: each rank's packed codes, 8-bit
    constants and second-level scales are contiguous slices of the whole
    matrix's, at element offset r0 * K."""
    if K <= 0 or K % 64:
        raise ValueError("K must be a positive multiple of 64")
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank out of range")
    group = 64 * 256
    step = group // _gcd(K, group)           # rows per whole number of groups
    units = -(-N // step)                    # the last unit may be short (the matrix's last group)
    u0, u1 = units * rank // world, units * (rank + 1) // world
    return min(N, u0 * step), min(N, u1 * step)


def _gcd(a: int, b: int) -> int:
    while b:
        a, b = b, a % b
    return a
