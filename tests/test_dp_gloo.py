"""World-size-2 gloo test (CPU) of the data-parallel exchange step: the
adapter gradients of every linear are summed across ranks."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bit_quantized_lora_blockwise_b200.dp import allreduce_adapter_grads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        g = torch.Generator().manual_seed(100 + rank)
        dA = torch.randn(64, 8, generator=g).to(torch.bfloat16)
        dB = torch.randn(8, 128, generator=g).to(torch.bfloat16)
        dA2 = torch.randn(32, 8, generator=g).to(torch.bfloat16)
        mine = [t.clone() for t in (dA, dB, dA2)]
        allreduce_adapter_grads([dA, dB, dA2])
        q.put((rank, [t.float() for t in mine], [t.float() for t in (dA, dB, dA2)]))
    finally:
        dist.destroy_process_group()


def test_adapter_grad_allreduce_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        rank, mine, summed = q.get(timeout=120)
        out[rank] = (mine, summed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for i in range(3):
        want = (out[0][0][i] + out[1][0][i]).to(torch.bfloat16).float()
        assert torch.equal(out[0][1][i], want)
        assert torch.equal(out[1][1][i], want)
