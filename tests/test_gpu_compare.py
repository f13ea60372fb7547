"""Parity of the comparison design the benchmark times against the fused
layer: dequantize the weight to HBM, then multiply with the library GEMM
(cuBLAS through torch) — the "dequantize, use, discard" order the pages
describe (intvml.com "DL0087 QLoRA", opening paragraph) — in both 16-bit
compute types (systemoverflow.com "QLoRA ... at Extreme Scale"). Its
outputs are checked against the oracle like the fused layer's, so the
timing comparison is between two correct implementations.
"""
import numpy as np
import pytest
import torch

import oracle
from bench import dequant_then_library
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, normal_bf16, normal_f16, weight_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _rel(got, want) -> float:
    g = got.float().cpu().numpy().astype(np.float64)
    den = np.max(np.abs(want))
    return float(np.max(np.abs(g - want)) / (den if den > 0 else 1.0))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("M,N,K,r", [(256, 1024, 512, 64), (40, 512, 1024, 8)])
def test_dequant_then_library_matches_oracle(dtype, M, N, K, r):
    W = weight_bf16(N, K, 0.02, 81 + M, 0.001)
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W))
    q_o, s2_o = oracle.double_quant(am_o)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    gen = normal_bf16 if dtype == torch.bfloat16 else normal_f16
    # adapters at N(0, 1/r): the low-rank term is as large as the base term
    X, A, B, dY = (gen(s, sd, 90 + i) for i, (s, sd) in
                   enumerate((((M, K), 1.0), ((K, r), r ** -0.5), ((r, N), r ** -0.5), ((M, N), 1.0))))
    Y, dX, dA, dB = dequant_then_library(pk, q, s2, X.cuda(), A.cuda(), B.cuda(), dY.cuda(), 16.0, N, K)
    torch.cuda.synchronize()
    if dtype == torch.bfloat16:
        wq = oracle.dequant(pk_o, q_o, s2_o, N * K).reshape(N, K)
        Xh, Ah, Bh, dYh = map(bf16_bits, (X, A, B, dY))
    else:
        wq = oracle.dequant_f16(pk_o, q_o, s2_o, N * K).reshape(N, K).view(np.float16)
        Xh, Ah, Bh, dYh = (t.numpy() for t in (X, A, B, dY))
    Yo, _ = oracle.linear_fwd(Xh, wq, Ah, Bh, 16.0, r)
    dXo, dAo, dBo = oracle.linear_bwd(Xh, dYh, wq, Ah, Bh, 16.0, r)
    for name, got, want in (("Y", Y, Yo), ("dX", dX, dXo), ("dA", dA, dAo), ("dB", dB, dBo)):
        assert got.dtype == dtype
        rel = _rel(got, want)
        assert rel <= TOL, f"{name}: max rel error {rel:.3e}"
