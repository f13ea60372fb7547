"""GPU parity of the fp16 compute type (systemoverflow.com "QLoRA: Efficient
Finetuning of Quantized LLMs at Extreme Scale": the adapters and the
computation run in 16-bit float or bfloat16).

The packed state is the same for both types; with fp16 the weight decodes
to W'[e] = f16_rne(L[code] * c') and every 16-bit operand and output is
fp16. Checked against the oracle (fp16 dequantization, fp64 layer):

* the standalone fp16 dequantization bit-exact, with ordinary, overflowing
  (beyond 65504 -> inf) and subnormal decoded magnitudes;
* the in-mainloop and in-register decode bit-exact through one-hot rows of
  X with B = 0 (each output row is then a column of W' exactly);
* the layer forward and backward within the layer tolerance on every path
  (few-token stream, 32-token tiles, 256-token CTA pairs with one and two
  sub-tiles, split K), and the adapter term alone (W' == 0) so that the
  fp16 low-rank steps are compared in their own right.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, f16_bits, normal_f16, weight_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rel(got, want) -> float:
    den = np.max(np.abs(want))
    return float(np.max(np.abs(_f64(got) - want)) / (den if den > 0 else 1.0))


def _state(W):
    N, K = W.shape
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W))
    q_o, s2_o = oracle.double_quant(am_o)
    wq = oracle.dequant_f16(pk_o, q_o, s2_o, N * K).reshape(N, K)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    return pk, q, s2, wq


@pytest.mark.parametrize("std", [0.02, 1.0e4, 2.0e-6])
def test_dequant_f16_bit_exact(std):
    N, K = 192, 1600  # second-level groups straddle rows
    W = weight_bf16(N, K, std, 21, 0.01)
    pk, q, s2, wq = _state(W)
    got = binding.dequant(pk, q, s2, N, K, dtype=torch.float16)
    torch.cuda.synchronize()
    assert got.dtype == torch.float16
    gb = f16_bits(got)
    assert np.array_equal(gb, wq)
    if std > 1e3:
        assert np.any((gb & 0x7FFF) == 0x7C00), "some decoded weights must overflow to inf"
    if std < 1e-5:
        assert np.any(((gb & 0x7C00) == 0) & ((gb & 0x03FF) != 0)), "some must be fp16 subnormals"


def _inputs(M, N, K, r, seed, sa=0.05, sb=0.05):
    X = normal_f16((M, K), 1.0, seed + 1)
    A = normal_f16((K, r), sa, seed + 2)
    B = normal_f16((r, N), sb, seed + 3)
    dY = normal_f16((M, N), 1.0, seed + 4)
    return X, A, B, dY


def _layer(M, N, K, r, pk, q, s2, wq, X, A, B, dY, alpha=16.0):
    Xd, Ad, Bd, dYd = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    XA = torch.empty((M, r), dtype=torch.float16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, Xd, Ad, Bd, alpha, N, K, XA_out=XA)
    dX, dA, dB = binding.linear_bwd(pk, q, s2, Xd, dYd, Ad, Bd, alpha, N, K, XA=XA)
    dX2, _, dB2 = binding.linear_bwd(pk, q, s2, Xd, dYd, Ad, Bd, alpha, N, K, XA=None)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    for t in (Y, XA, dX, dA, dB):
        assert t.dtype == torch.float16
    w = wq.view(np.float16)
    Xh, Ah, Bh, dYh = (t.numpy() for t in (X, A, B, dY))
    Yo, XAo = oracle.linear_fwd(Xh, w, Ah, Bh, alpha, r)
    dXo, dAo, dBo = oracle.linear_bwd(Xh, dYh, w, Ah, Bh, alpha, r)
    return {"Y": (Y, Yo), "XA": (XA, XAo), "dX": (dX, dXo), "dA": (dA, dAo), "dB": (dB, dBo),
            "dX_recompute": (dX2, dXo), "dB_recompute": (dB2, dBo)}


# (M, N, K, r): few-token stream (M <= 16), 32-token tiles, CTA pairs with one
# and two 256-token sub-tiles, split K
SHAPES = [(1, 1024, 2048, 64), (16, 512, 1024, 16), (24, 1024, 2048, 128), (300, 512, 1024, 64),
          (1300, 576, 640, 32), (2048, 256, 4096, 64)]


@pytest.mark.parametrize("M,N,K,r", SHAPES)
def test_layer_f16(M, N, K, r):
    W = weight_bf16(N, K, 0.02, 31 + M, 0.001)
    pk, q, s2, wq = _state(W)
    res = _layer(M, N, K, r, pk, q, s2, wq, *_inputs(M, N, K, r, 40 + M))
    for name, (got, want) in res.items():
        rel = _rel(got, want)
        assert rel <= TOL, f"{name}: max rel error {rel:.3e}"


@pytest.mark.parametrize("M,N,K,r", [(3, 512, 1024, 64), (24, 1024, 512, 8), (300, 512, 1024, 128),
                                     (1300, 512, 512, 64)])
def test_adapter_term_alone_f16(M, N, K, r):
    """Every code is the zero level, so W' == 0 and Y = s (X A) B, dX = s (dY B^T) A^T."""
    nb = N * K // 64
    g = torch.Generator().manual_seed(M + N)
    pk = torch.full((N * K // 2,), 0x77, dtype=torch.uint8)
    q = torch.randint(1, 256, (nb,), generator=g, dtype=torch.int64).to(torch.uint8)
    s2 = (torch.rand(((nb + 255) // 256,), generator=g) * 0.5 + 0.01).to(torch.float32)
    wq = oracle.dequant_f16(pk.numpy(), q.numpy(), s2.numpy(), N * K).reshape(N, K)
    assert not np.any(wq)
    X, A, B, dY = _inputs(M, N, K, r, 50 + M, sa=0.3, sb=0.3)
    res = _layer(M, N, K, r, pk.cuda(), q.cuda(), s2.cuda(), wq, X, A, B, dY)
    for name in ("Y", "dX", "dX_recompute"):
        got, want = res[name]
        assert torch.count_nonzero(got).item() > got.numel() // 2, name
        rel = _rel(got, want)
        assert rel <= TOL, f"{name}: max rel error {rel:.3e}"


@pytest.mark.parametrize("M", [5, 24, 300, 1100])
def test_one_hot_rows_give_columns_of_w_f16(M):
    N, K, r = 512, 1024, 16
    W = weight_bf16(N, K, 0.02, 61, 0.001)
    pk, q, s2, wq = _state(W)
    ks = (np.arange(M) * 37 + 5) % K
    Xh = torch.zeros((M, K), dtype=torch.float16)
    Xh[np.arange(M), ks] = 1.0
    A = normal_f16((K, r), 0.05, 62).cuda()
    B = torch.zeros((r, N), dtype=torch.float16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, Xh.cuda(), A, B, 16.0, N, K)
    torch.cuda.synchronize()
    assert np.array_equal(f16_bits(Y), wq[:, ks].T)


def test_mixed_types_are_refused():
    N, K, r, M = 256, 256, 8, 4
    W = weight_bf16(N, K, 0.02, 71)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    X = normal_f16((M, K), 1.0, 72).cuda()
    A = normal_f16((K, r), 0.05, 73).cuda().to(torch.bfloat16)
    B = normal_f16((r, N), 0.05, 74).cuda()
    with pytest.raises(TypeError):
        binding.linear_fwd(pk, q, s2, X, A, B, 16.0, N, K)
