"""GPU parity of the fused QLoRA linear forward/backward against the float64
oracle.

Tolerance: max|y - y*| / max|y*| <= 1e-2 per output tensor (bf16 inputs,
fp32 accumulation, fp64 oracle fed the oracle's own dequantized weight).
Bit-exact pins of the in-mainloop dequantization: with B = 0, a one-hot row
of X (a single 1.0) makes the forward output row exactly a column of W', and
a one-hot row of dY makes the dX row exactly a row of W' (one nonzero
product, accumulated in fp32, rounded to bf16 = the bf16 weight itself).
B = 0 gives dA = 0 and A = 0 gives dB = 0 exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import weight_bf16, normal_bf16, bf16_bits

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _rel(got: torch.Tensor, want: np.ndarray) -> float:
    g = got.float().cpu().numpy().astype(np.float64)
    den = np.max(np.abs(want))
    return float(np.max(np.abs(g - want)) / (den if den > 0 else 1.0))


class Layer:
    def __init__(self, M, N, K, r, alpha=16.0, seed=0, w_std=0.02, outl=0.0, zero_B=False, zero_A=False):
        self.M, self.N, self.K, self.r, self.alpha = M, N, K, r, alpha
        self.W = weight_bf16(N, K, w_std, seed + 1, outl)
        self.X = normal_bf16((M, K), 1.0, seed + 2)
        self.A = normal_bf16((K, r), 0.01, seed + 3) * (0 if zero_A else 1)
        self.B = normal_bf16((r, N), 0.01, seed + 4) * (0 if zero_B else 1)
        self.dY = normal_bf16((M, N), 1.0, seed + 5)
        bits = bf16_bits(self.W)
        pk, am = oracle.quantize_nf4(bits)
        q, s2 = oracle.double_quant(am)
        self.Wq_bits = oracle.dequant(pk, q, s2, N * K).reshape(N, K)
        Wc = self.W.cuda()
        self.pk, am_g = binding.quantize_nf4(Wc)
        self.q, self.s2 = binding.double_quant(am_g)

    def gpu(self, t):
        return t.cuda()

    def fwd(self, XA_out=True):
        XA = torch.empty((self.M, self.r), dtype=torch.bfloat16, device="cuda") if XA_out else None
        Y = binding.linear_fwd(self.pk, self.q, self.s2, self.X.cuda(), self.A.cuda(), self.B.cuda(),
                               self.alpha, self.N, self.K, XA_out=XA)
        return Y, XA

    def bwd(self, XA=None):
        return binding.linear_bwd(self.pk, self.q, self.s2, self.X.cuda(), self.dY.cuda(), self.A.cuda(),
                                  self.B.cuda(), self.alpha, self.N, self.K, XA=XA)

    def oracle_fwd(self):
        return oracle.linear_fwd(bf16_bits(self.X), self.Wq_bits, bf16_bits(self.A), bf16_bits(self.B),
                                 self.alpha, self.r)

    def oracle_bwd(self):
        return oracle.linear_bwd(bf16_bits(self.X), bf16_bits(self.dY), self.Wq_bits, bf16_bits(self.A),
                                 bf16_bits(self.B), self.alpha, self.r)


@pytest.mark.parametrize("M,N,K,r", [
    (16, 1024, 1024, 8),     # single-linear workload (r = 8, alpha = 16)
    (3, 192, 320, 8),        # ragged: M tail, N % 128 == 64, K/64 odd
    (300, 256, 512, 64),     # M spans two 256-column tiles with a tail
    (520, 384, 256, 16),     # three row tiles, K = 256
    (64, 128, 128, 128),     # rank 128
    (40, 256, 192, 256),     # rank 256 (four low-rank K blocks)
    (2048, 4096, 512, 16),   # forward without split (512-token tiles of two sub-tiles)
    (2048, 512, 4096, 16),   # backward without split
    (1300, 768, 640, 32),    # two sub-tiles with a ragged last tile (276 tokens: the peer's half partly empty), split K
    (1030, 256, 1536, 64),   # two sub-tiles, last tile of 6 tokens, split K
])
def test_fwd_bwd_parity(M, N, K, r):
    L = Layer(M, N, K, r, seed=M * 7 + N + K + r)
    Y, XA = L.fwd()
    dX, dA, dB = L.bwd(XA)
    dX2, dA2, dB2 = L.bwd(None)  # recompute XA inside the backward
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    Yo, XAo = L.oracle_fwd()
    dXo, dAo, dBo = L.oracle_bwd()
    assert _rel(Y, Yo) <= TOL
    assert _rel(XA, XAo) <= TOL
    assert _rel(dX, dXo) <= TOL
    assert _rel(dA, dAo) <= TOL
    assert _rel(dB, dBo) <= TOL
    assert torch.equal(dX, dX2) and torch.equal(dA, dA2)
    assert _rel(dB2, dBo) <= TOL


def test_one_hot_rows_pin_in_mainloop_dequant():
    M, N, K, r = 192, 256, 384, 8
    L = Layer(M, N, K, r, seed=5, outl=0.001, zero_B=True)
    ks = (np.arange(M) * 37) % K
    X = torch.zeros((M, K), dtype=torch.bfloat16)
    X[np.arange(M), ks] = 1.0
    L.X = X
    Y, _ = L.fwd()
    ns = (np.arange(M) * 53) % N
    dY = torch.zeros((M, N), dtype=torch.bfloat16)
    dY[np.arange(M), ns] = 1.0
    L.dY = dY
    dX, dA, dB = L.bwd(None)
    torch.cuda.synchronize()
    Wq = L.Wq_bits
    assert np.array_equal(bf16_bits(Y), Wq[:, ks].T), "forward row = column of W'"
    assert np.array_equal(bf16_bits(dX), Wq[ns, :]), "backward row = row of W'"
    assert torch.count_nonzero(dA).item() == 0  # B = 0 -> G = 0 -> dA = 0


def test_zero_adapters():
    L = Layer(64, 256, 256, 16, seed=11, zero_B=True)
    Y, XA = L.fwd()
    dX, dA, dB = L.bwd(XA)
    Yo, _ = L.oracle_fwd()
    assert _rel(Y, Yo) <= TOL
    assert torch.count_nonzero(dA).item() == 0
    L = Layer(64, 256, 256, 16, seed=12, zero_A=True)
    Y, XA = L.fwd()
    dX, dA, dB = L.bwd(XA)
    assert torch.count_nonzero(XA).item() == 0
    assert torch.count_nonzero(dB).item() == 0


def test_packed_weight_untouched_by_backward():
    L = Layer(128, 256, 256, 16, seed=21)
    before = (L.pk.clone(), L.q.clone(), L.s2.clone())
    Y, XA = L.fwd()
    L.bwd(XA)
    torch.cuda.synchronize()
    assert torch.equal(before[0], L.pk) and torch.equal(before[1], L.q) and torch.equal(before[2], L.s2)


@pytest.mark.parametrize("M", [1, 4, 16, 17, 24, 32])
def test_small_m_split_k(M):
    """Few tokens. M <= 16: the register-dequant weight stream; 16 < M <= 32:
    the fused GEMM on 32-token tiles, K split across CTAs (fp32 partials +
    reduce). The backward always takes the fused GEMM."""
    L = Layer(M, 1024, 2048, 64, seed=100 + M, w_std=0.015)
    Y, XA = L.fwd()
    Yo, XAo = L.oracle_fwd()
    assert _rel(Y, Yo) <= TOL
    assert _rel(XA, XAo) <= TOL
    dX, dA, dB = L.bwd(XA)
    dXo, dAo, dBo = L.oracle_bwd()
    assert _rel(dX, dXo) <= TOL and _rel(dA, dAo) <= TOL and _rel(dB, dBo) <= TOL


@pytest.mark.parametrize("M,N,K,r", [
    (16, 4096, 4096, 64),   # bands shared by two CTAs (stream-K pieces)
    (1, 8192, 2048, 64),    # one token
    (7, 2112, 1600, 16),    # half band at the end of N, one-block K chunk at the end of K
    (12, 1024, 8192, 8),    # long K: many chunks per band
])
def test_few_token_forward_stream_k(M, N, K, r):
    """Few tokens: the forward streams the packed weight once, dequantizing
    in registers; bands split across CTAs are summed in a fixed order, so two
    calls give the same bits."""
    L = Layer(M, N, K, r, seed=300 + M + N + K, w_std=0.015, outl=0.001)
    Y, XA = L.fwd()
    Y2, XA2 = L.fwd()
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    Yo, XAo = L.oracle_fwd()
    assert _rel(Y, Yo) <= TOL
    assert _rel(XA, XAo) <= TOL
    assert torch.equal(Y, Y2) and torch.equal(XA, XA2)


def test_few_token_one_hot_rows_pin_register_dequant():
    """B = 0 and one-hot rows of X: each forward row is exactly a column of
    W', which pins the in-register dequantization of the few-token path."""
    M, N, K, r = 16, 2112, 1600, 8
    L = Layer(M, N, K, r, seed=77, outl=0.001, zero_B=True)
    ks = (np.arange(M) * 97 + 13) % K
    X = torch.zeros((M, K), dtype=torch.bfloat16)
    X[np.arange(M), ks] = 1.0
    L.X = X
    Y, _ = L.fwd()
    torch.cuda.synchronize()
    assert np.array_equal(bf16_bits(Y), L.Wq_bits[:, ks].T)
