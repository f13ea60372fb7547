"""Decoder-block chaining (promptingindex.com "QLoRA: Finetuning 65B Models on
a Single GPU", "LoRA placement": adapters on every linear; systemoverflow.com
"QLoRA ... at Extreme Scale": gradient checkpointing): qlora_block_fwd /
qlora_block_bwd run the seven linears of a LLaMA-shaped block (q, k, v, o,
gate, up, down) in one call over two streams.

Every kernel is deterministic, so the block's outputs must be bit-identical
to the same linears run one by one on one stream, for both recompute
schedules (X A saved by the forward, or recomputed by the backward), on the
few-token path and on the CTA-pair path, and in fp16; the block is also
captured into a CUDA graph whose replay must reproduce the eager results.
One linear is compared with the oracle as well.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, normal_bf16, weight_bf16

pytestmark = pytest.mark.gpu
D, FFN = 512, 1408  # q, k, v, o: D x D; gate, up: FFN x D; down: D x FFN


def _block(M, r, dtype, seed=1):
    shapes = [(D, D)] * 4 + [(FFN, D), (FFN, D), (D, FFN)]
    out = []
    for i, (N, K) in enumerate(shapes):
        W = weight_bf16(N, K, 0.02, seed + 10 * i, 0.001)
        pk, am = binding.quantize_nf4(W.cuda())
        q, s2 = binding.double_quant(am)

        def t(shape, sd, k):
            return normal_bf16(shape, sd, seed + 10 * i + k).to(dtype).cuda()
        out.append({"packed": pk, "q": q, "scale2": s2, "N": N, "K": K, "W": W,
                    "X": t((M, K), 1.0, 1), "A": t((K, r), 0.05, 2), "B": t((r, N), 0.05, 3),
                    "dY": t((M, N), 1.0, 4),
                    "Y": torch.empty((M, N), dtype=dtype, device="cuda"),
                    "XA": torch.empty((M, r), dtype=dtype, device="cuda"),
                    "dX": torch.empty((M, K), dtype=dtype, device="cuda"),
                    "dA": torch.empty((K, r), dtype=dtype, device="cuda"),
                    "dB": torch.empty((r, N), dtype=dtype, device="cuda")})
    return out


def _one_by_one(lins, alpha, save_xa):
    res = []
    for L in lins:
        XA = torch.empty_like(L["XA"]) if save_xa else None
        Y = binding.linear_fwd(L["packed"], L["q"], L["scale2"], L["X"], L["A"], L["B"], alpha, L["N"], L["K"],
                               XA_out=XA)
        dX, dA, dB = binding.linear_bwd(L["packed"], L["q"], L["scale2"], L["X"], L["dY"], L["A"], L["B"], alpha,
                                        L["N"], L["K"], XA=XA)
        res.append((Y, XA, dX, dA, dB))
    return res


def _assert_same(lins, ref, save_xa):
    for L, (Y, XA, dX, dA, dB) in zip(lins, ref):
        assert torch.equal(L["Y"], Y)
        if save_xa:
            assert torch.equal(L["XA"], XA)
        assert torch.equal(L["dX"], dX)
        assert torch.equal(L["dA"], dA)
        assert torch.equal(L["dB"], dB)


@pytest.mark.parametrize("M,save_xa,dtype", [(256, True, torch.bfloat16), (256, False, torch.bfloat16),
                                             (8, True, torch.bfloat16), (1100, True, torch.float16),
                                             (40, False, torch.float16)])
def test_block_equals_linears_one_by_one(M, save_xa, dtype):
    r, alpha = 16, 16.0
    lins = _block(M, r, dtype)
    ref = _one_by_one(lins, alpha, save_xa)
    ws = binding.block_fwd(lins, M, r, alpha, save_xa=save_xa)
    binding.block_bwd(lins, M, r, alpha, save_xa=save_xa, workspace=ws)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    _assert_same(lins, ref, save_xa)


def test_block_linear_against_oracle():
    M, r, alpha = 256, 16, 16.0
    lins = _block(M, r, torch.bfloat16, seed=5)
    ws = binding.block_fwd(lins, M, r, alpha)
    torch.cuda.synchronize()
    L = lins[6]  # down: N = D, K = FFN
    pk, am = oracle.quantize_nf4(bf16_bits(L["W"]))
    q, s2 = oracle.double_quant(am)
    wq = oracle.dequant(pk, q, s2, L["N"] * L["K"]).reshape(L["N"], L["K"])
    Yo, _ = oracle.linear_fwd(bf16_bits(L["X"]), wq, bf16_bits(L["A"]), bf16_bits(L["B"]), alpha, r)
    y = L["Y"].float().cpu().numpy().astype(np.float64)
    assert np.max(np.abs(y - Yo)) / np.max(np.abs(Yo)) <= 1e-2
    del ws


def test_block_in_a_cuda_graph():
    M, r, alpha = 256, 16, 16.0
    lins = _block(M, r, torch.bfloat16, seed=9)
    ws = binding.block_fwd(lins, M, r, alpha)          # uncaptured call: sets up kernels and streams
    binding.block_bwd(lins, M, r, alpha, workspace=ws)
    torch.cuda.synchronize()
    ref = [tuple(L[k].clone() for k in ("Y", "XA", "dX", "dA", "dB")) for L in lins]
    for L in lins:
        for k in ("Y", "XA", "dX", "dA", "dB"):
            L[k].zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        binding.block_fwd(lins, M, r, alpha, workspace=ws)
        binding.block_bwd(lins, M, r, alpha, workspace=ws)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    for L, want in zip(lins, ref):
        for k, w in zip(("Y", "XA", "dX", "dA", "dB"), want):
            assert torch.equal(L[k], w), k
    del g
