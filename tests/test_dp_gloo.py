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


# --- the data-parallel step and the codec split, composed on CPU ranks ----
import numpy as np  # noqa: E402

import oracle  # noqa: E402
from bit_quantized_lora_blockwise_b200.dp import codec_shard_rows, token_shard  # noqa: E402
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, normal_bf16, weight_bf16  # noqa: E402

M_ALL, N, K, R, ALPHA = 40, 128, 192, 8, 16.0


def _layer_inputs():
    W = weight_bf16(N, K, 0.02, 7)
    pk, am = oracle.quantize_nf4(bf16_bits(W))
    q, s2 = oracle.double_quant(am)
    wq = oracle.dequant(pk, q, s2, N * K).reshape(N, K)
    X, A, B, dY = (bf16_bits(normal_bf16(s, sd, 20 + i)) for i, (s, sd) in
                   enumerate((((M_ALL, K), 1.0), ((K, R), 0.05), ((R, N), 0.05), ((M_ALL, N), 1.0))))
    return wq, X, A, B, dY


def _dp_worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wq, X, A, B, dY = _layer_inputs()
        t0, t1 = token_shard(M_ALL, rank, world)
        _, dA, dB = oracle.linear_bwd(X[t0:t1], dY[t0:t1], wq, A, B, ALPHA, R)
        g = [torch.from_numpy(dA.astype(np.float32)), torch.from_numpy(dB.astype(np.float32))]
        allreduce_adapter_grads(g)
        # codec: this rank's rows of a weight, in whole second-level groups
        Wc = weight_bf16(320, 448, 0.02, 9)  # K = 448: a group spans 36 4/7 rows
        r0, r1 = codec_shard_rows(320, 448, rank, world)
        part = None
        if r1 > r0:
            pk, am = oracle.quantize_nf4(bf16_bits(Wc[r0:r1]))
            qq, s2 = oracle.double_quant(am)
            part = (r0, r1, pk, qq, s2)
        q.put((rank, [t.numpy() for t in g], part))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_dp_step_and_codec_split(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        rank, g, part = q.get(timeout=180)
        out[rank] = (g, part)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the all-reduced shard gradients are the whole batch's (dA, dB are sums over tokens)
    wq, X, A, B, dY = _layer_inputs()
    _, dA, dB = oracle.linear_bwd(X, dY, wq, A, B, ALPHA, R)
    for rank in range(world):
        gA, gB = out[rank][0]
        np.testing.assert_allclose(gA, dA, rtol=1e-5, atol=1e-6 * np.abs(dA).max())
        np.testing.assert_allclose(gB, dB, rtol=1e-5, atol=1e-6 * np.abs(dB).max())
    # the codec shards, concatenated in rank order, are the whole matrix's codec, bit for bit
    Wc = weight_bf16(320, 448, 0.02, 9)
    pk, am = oracle.quantize_nf4(bf16_bits(Wc))
    qq, s2 = oracle.double_quant(am)
    parts = [out[r][1] for r in range(world) if out[r][1] is not None]
    assert parts[0][0] == 0 and parts[-1][1] == 320
    assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    assert np.array_equal(np.concatenate([p[2] for p in parts]), pk)
    assert np.array_equal(np.concatenate([p[3] for p in parts]), qq)
    assert np.array_equal(np.concatenate([p[4] for p in parts]).view(np.uint32), s2.view(np.uint32))


def test_codec_shard_rows_whole_groups():
    for N, K in ((4096, 4096), (11008, 4096), (4096, 11008), (320, 448), (100, 64)):
        for world in (1, 2, 3, 8):
            spans = [codec_shard_rows(N, K, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == N
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            for r0, _ in spans:
                assert (r0 * K) % (64 * 256) == 0 or r0 == N
    assert [token_shard(10, r, 3) for r in range(3)] == [(0, 3), (3, 6), (6, 10)]
