"""GPU parity of the codec and the fused layer with the alternative code
tables (4-bit integers, the E2M1 4-bit float, and the signed-linear and
dynamic-exponent 8-bit constant maps), which the pages compare with NF4
(promptingindex.com "Finetuning 65B Models on a Single GPU", section "4-bit
NormalFloat"). The tables are ordinary inputs of the calls, so these tests
check that nothing in the kernels assumes the NF4 or k/255 values:

* codes, constants and the dequantized weight bit-exact against the oracle
  for every pair of a 4-bit table and an 8-bit map (the quantizer's bucketed
  encode and the double quant's bucketed or binary-search encode are chosen
  per table by the library);
* the fused forward and backward within the layer tolerance, and one-hot
  rows (B = 0) that make the forward output exactly the columns of the
  dequantized weight, so the in-mainloop decode is pinned bit for bit with
  the alternative tables too.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
from oracle import codebooks as cb
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, normal_bf16, weight_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-2

TABLES4 = {"nf4": oracle.nf4_levels, "int4": cb.int4_levels, "fp4": cb.fp4_levels}
TABLES8 = {"linear": oracle.dq_levels, "signed": cb.dq_signed_levels, "dynamic": cb.dq_dynamic_levels}


def _rel(got, want) -> float:
    g = got.float().cpu().numpy().astype(np.float64)
    den = np.max(np.abs(want))
    return float(np.max(np.abs(g - want)) / (den if den > 0 else 1.0))


@pytest.mark.parametrize("t4,t8", list(itertools.product(TABLES4, TABLES8)))
def test_codec_bit_exact_with_alternative_tables(t4, t8):
    lv, tt = TABLES4[t4](), TABLES8[t8]()
    N, K = 192, 1600  # 25 blocks per row: second-level groups straddle rows
    W = weight_bf16(N, K, 0.02, 31, 0.002)
    bits = bf16_bits(W)
    pk_o, am_o = oracle.quantize_nf4(bits, lv)
    q_o, s2_o = oracle.double_quant(am_o, tt)
    wq_o = oracle.dequant(pk_o, q_o, s2_o, N * K, lv, tt)
    pk, am = binding.quantize_nf4(W.cuda(), nf4=lv)
    q, s2 = binding.double_quant(am, t8=tt)
    wq = binding.dequant(pk, q, s2, N, K, nf4=lv, t8=tt)
    torch.cuda.synchronize()
    assert np.array_equal(pk.cpu().numpy(), pk_o)
    assert np.array_equal(am.cpu().numpy().view(np.uint32), am_o.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_o.view(np.uint32))
    assert np.array_equal(bf16_bits(wq).reshape(-1), wq_o)


@pytest.mark.parametrize("t4,t8,M", [("int4", "dynamic", 300), ("fp4", "signed", 24), ("int4", "linear", 8)])
def test_fused_layer_with_alternative_tables(t4, t8, M):
    lv, tt = TABLES4[t4](), TABLES8[t8]()
    N, K, r, alpha = 512, 1024, 16, 16.0
    W = weight_bf16(N, K, 0.02, 41, 0.001)
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W), lv)
    q_o, s2_o = oracle.double_quant(am_o, tt)
    wq = oracle.dequant(pk_o, q_o, s2_o, N * K, lv, tt).reshape(N, K)
    pk, am = binding.quantize_nf4(W.cuda(), nf4=lv)
    q, s2 = binding.double_quant(am, t8=tt)
    X, A, B, dY = (normal_bf16(s, sd, 42 + i) for i, (s, sd) in
                   enumerate((((M, K), 1.0), ((K, r), 0.05), ((r, N), 0.05), ((M, N), 1.0))))
    XA = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, X.cuda(), A.cuda(), B.cuda(), alpha, N, K, nf4=lv, t8=tt, XA_out=XA)
    dX, dA, dB = binding.linear_bwd(pk, q, s2, X.cuda(), dY.cuda(), A.cuda(), B.cuda(), alpha, N, K, XA=XA,
                                    nf4=lv, t8=tt)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    Xb, Ab, Bb, dYb = map(bf16_bits, (X, A, B, dY))
    Yo, _ = oracle.linear_fwd(Xb, wq, Ab, Bb, alpha, r)
    dXo, dAo, dBo = oracle.linear_bwd(Xb, dYb, wq, Ab, Bb, alpha, r)
    for name, got, want in (("Y", Y, Yo), ("dX", dX, dXo), ("dA", dA, dAo), ("dB", dB, dBo)):
        assert _rel(got, want) <= TOL, name

    # one-hot rows of X with B = 0: each output row is a column of W' exactly
    ks = (np.arange(M) * 37 + 5) % K
    Xh = torch.zeros((M, K), dtype=torch.bfloat16)
    Xh[np.arange(M), ks] = 1.0
    Y1 = binding.linear_fwd(pk, q, s2, Xh.cuda(), A.cuda(), torch.zeros_like(B).cuda(), alpha, N, K, nf4=lv, t8=tt)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(Y1), wq[:, ks].T)
