"""Parity at the workloads' full sizes, in the configuration bench.py times.

Inputs come from the same seeded generators as the benchmark
(bit_quantized_lora_blockwise_b200/inputs.py). The codec is compared bit for bit on whole
matrices. The GEMM outputs are compared on 256 seeded rows of Y and dX
(the oracle computes each sampled row in float64) and in full for XA, dA and
dB, which reduce over every token; the tolerance is the layer tolerance,
max|y - y*| / max|y*| <= 1e-2 per compared tensor.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import WORKLOADS, bf16_bits, layer_inputs

pytestmark = pytest.mark.gpu
TOL = 1e-2
NROWS = 256


def _rel(got, want) -> float:
    g = got.float().cpu().numpy().astype(np.float64) if torch.is_tensor(got) else got
    den = np.max(np.abs(want))
    return float(np.max(np.abs(g - want)) / (den if den > 0 else 1.0))


def _rows(M: int, seed: int) -> np.ndarray:
    if M <= NROWS:
        return np.arange(M)
    rng = np.random.default_rng(seed)
    pick = rng.choice(M - 2, NROWS - 2, replace=False) + 1
    return np.sort(np.concatenate([[0, M - 1], pick]))


def _oracle_weight(W: torch.Tensor):
    """(packed, absmax, q, scale2, dequantized bf16 bits [N, K]) from the oracle."""
    N, K = W.shape
    bits = bf16_bits(W)
    pk, am = oracle.quantize_nf4(bits)
    q, s2 = oracle.double_quant(am)
    wq = oracle.dequant(pk, q, s2, N * K).reshape(N, K)
    return pk, am, q, s2, wq


def test_codec_13b_ffn_weight_bit_exact(cuda_device):
    wl = WORKLOADS["llama13b_quant_sweep"]
    li = 4  # gate: 5120 -> 13824, 70.8 M weights
    W = layer_inputs(wl, li, 0)["W"]
    N, K = W.shape
    pk_o, am_o, q_o, s2_o, wq_o = _oracle_weight(W)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    wq = binding.dequant(pk, q, s2, N, K)
    torch.cuda.synchronize()
    assert np.array_equal(pk.cpu().numpy(), pk_o)
    assert np.array_equal(am.cpu().numpy().view(np.uint32), am_o.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_o.view(np.uint32))
    assert np.array_equal(bf16_bits(wq), wq_o)


def _check_linear(wl, li, M, recompute_xa=False):
    inp = layer_inputs(wl, li, M)
    W, X, A, B, dY = (inp[k] for k in ("W", "X", "A", "B", "dY"))
    N, K = W.shape
    r, alpha = wl.r, wl.alpha
    _, _, _, _, wq = _oracle_weight(W)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    Xd, Ad, Bd, dYd = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    XA = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, Xd, Ad, Bd, alpha, N, K, XA_out=XA)
    dX, dA, dB = binding.linear_bwd(pk, q, s2, Xd, dYd, Ad, Bd, alpha, N, K, XA=None if recompute_xa else XA)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    rows = _rows(M, 1000 * li + M)
    Xb, Ab, Bb, dYb = map(bf16_bits, (X, A, B, dY))
    Yo = oracle.linear_fwd_rows(rows, Xb, wq, Ab, Bb, alpha, r)
    assert _rel(Y.float().cpu().numpy()[rows].astype(np.float64), Yo) <= TOL
    XAo = oracle.bf16_bits_to_f64(Xb) @ oracle.bf16_bits_to_f64(Ab)
    assert _rel(XA, XAo) <= TOL
    dXo, dAo, dBo = oracle.linear_bwd_rows(rows, Xb, dYb, wq, Ab, Bb, alpha, r)
    assert _rel(dX.float().cpu().numpy()[rows].astype(np.float64), dXo) <= TOL
    assert _rel(dA, dAo) <= TOL
    assert _rel(dB, dBo) <= TOL


@pytest.mark.parametrize("li", [4, 6])  # gate 4096 -> 11008, down 11008 -> 4096
def test_llama7b_linear_full_size(cuda_device, li):
    _check_linear(WORKLOADS["llama7b_set"], li, 2048)


def test_llama33b_down_full_size_recompute_xa(cuda_device):
    # down projection 17920 -> 6656, batch 1 x 2048 tokens, X A recomputed in the backward
    _check_linear(WORKLOADS["llama33b_block"], 6, 2048, recompute_xa=True)


@pytest.mark.parametrize("li,M", [(0, 1), (0, 4), (0, 16), (4, 1)])  # q 8192^2; gate 8192 -> 22016
def test_llama65b_few_token_forward_full_size(cuda_device, li, M):
    wl = WORKLOADS["llama65b_fwd"]
    inp = layer_inputs(wl, li, M, need_grad_inputs=False)
    W, X, A, B = (inp[k] for k in ("W", "X", "A", "B"))
    N, K = W.shape
    _, _, _, _, wq = _oracle_weight(W)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    XA = torch.empty((M, wl.r), dtype=torch.bfloat16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, X.cuda(), A.cuda(), B.cuda(), wl.alpha, N, K, XA_out=XA)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    Yo, XAo = oracle.linear_fwd(bf16_bits(X), wq, bf16_bits(A), bf16_bits(B), wl.alpha, wl.r)
    assert _rel(Y, Yo) <= TOL
    assert _rel(XA, XAo) <= TOL


@pytest.mark.parametrize("li", [0, 4, 6])  # q 4096^2, gate 4096 -> 11008, down 11008 -> 4096
def test_llama7b_every_output_against_dequant_then_fp32_matmul(cuda_device, li):
    """Every element of Y, dX, dA and dB at full size (M = 2048), against the
    dequantize-then-multiply formulation computed with fp32 matmuls on the
    device, from the library's own dequantized W' (bit-exact to the oracle
    by the codec tests). Complements the fp64 oracle's sampled rows above."""
    wl = WORKLOADS["llama7b_set"]
    M = 2048
    inp = layer_inputs(wl, li, M)
    W, X, A, B, dY = (inp[k].cuda() for k in ("W", "X", "A", "B", "dY"))
    N, K = W.shape
    r, alpha = wl.r, wl.alpha
    s = alpha / r
    pk, am = binding.quantize_nf4(W)
    q, s2 = binding.double_quant(am)
    wq = binding.dequant(pk, q, s2, N, K)
    XA = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, X, A, B, alpha, N, K, XA_out=XA)
    dX, dA, dB = binding.linear_bwd(pk, q, s2, X, dY, A, B, alpha, N, K, XA=XA)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    tf32 = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        Xf, Wf, Af, Bf, dYf = X.float(), wq.float(), A.float(), B.float(), dY.float()
        XAf = Xf @ Af
        Yr = Xf @ Wf.t() + s * (XAf @ Bf)
        G = dYf @ Bf.t()
        dXr = dYf @ Wf + s * (G @ Af.t())
        dAr = s * (Xf.t() @ G)
        dBr = s * (XAf.t() @ dYf)
    finally:
        torch.backends.cuda.matmul.allow_tf32 = tf32

    def rel(got, want):
        return float((got.float() - want).abs().max() / want.abs().max())

    assert rel(Y, Yr) <= TOL
    assert rel(XA, XAf) <= TOL
    assert rel(dX, dXr) <= TOL
    assert rel(dA, dAr) <= TOL
    assert rel(dB, dBr) <= TOL
