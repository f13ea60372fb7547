"""GPU parity of the rank-r adapter term of the fused QLoRA linear.

With the workloads' adapters, A, B ~ N(0, 0.01), the low-rank term
s (X A) B is about 1 % of the base term X W'^T or less, so a check of the
whole output at max|y - y*| / max|y*| <= 1e-2 cannot see it: a GEMM that
dropped its rank-r K-steps would pass. These tests make the adapter term
the part being compared (intvml.com "DL0087 QLoRA", Figure 1 and the
formulation's symbol list: the low-rank update, scaled by alpha / r, is
added to the frozen base's output; its gradient flows back through the
same product):

* W' == 0 exactly. Every packed code is the zero level (nibble 7) while the
  block constants are random and non-zero, so the in-mainloop decode must
  produce exact zeros and the outputs are the adapter products alone:
  Y = s (X A) B and dX = s (dY B^T) A^T.
* A real NF4 weight with A, B ~ N(0, 1): the adapter term is about a
  hundred times the base term.

Every case runs on the tile the library picks for it: the few-token
register stream (M <= 16), 32-token tiles (M <= 32), 256-token tiles, with
and without the split of K across CTAs, at r = 8, 64, 128 and 256. The
tolerance is the layer's, 1e-2 of the compared tensor's max. The elementwise
error |y - y*| / (|y*| + 1e-3 rms(y*)) is reported beside it (recorded as a
test property and printed); it is not a gate, since bf16 rounding of s X A
before its rank-r product (a reading the layer allows) makes it large
wherever the adapter sum cancels.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, normal_bf16, weight_bf16

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rel(got, want) -> float:
    den = np.max(np.abs(want))
    return float(np.max(np.abs(_f64(got) - want)) / (den if den > 0 else 1.0))


def _elem(got, want) -> float:
    floor = 1e-3 * np.sqrt(np.mean(want * want))
    return float(np.max(np.abs(_f64(got) - want) / (np.abs(want) + floor)))


def _zero_weight(N, K, seed):
    """Packed state whose every code is the zero level, with random non-zero
    8-bit constant codes and second-level scales."""
    g = torch.Generator().manual_seed(seed)
    nb = N * K // 64
    pk = torch.full((N * K // 2,), 0x77, dtype=torch.uint8)
    q = torch.randint(1, 256, (nb,), generator=g, dtype=torch.int64).to(torch.uint8)
    s2 = (torch.rand(((nb + 255) // 256,), generator=g) * 0.5 + 0.01).to(torch.float32)
    wq = oracle.dequant(pk.numpy(), q.numpy(), s2.numpy(), N * K).reshape(N, K)
    assert not np.any(wq), "the zero level must decode to +0 whatever the constant"
    return pk.cuda(), q.cuda(), s2.cuda(), wq


def _nf4_weight(N, K, seed):
    W = weight_bf16(N, K, 0.02, seed, 0.001)
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W))
    q_o, s2_o = oracle.double_quant(am_o)
    wq = oracle.dequant(pk_o, q_o, s2_o, N * K).reshape(N, K)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    return pk, q, s2, wq


def _run(M, N, K, r, weight, seed, record_property, alpha=16.0):
    pk, q, s2, wq = weight(N, K, seed)
    X = normal_bf16((M, K), 1.0, seed + 1)
    A = normal_bf16((K, r), 1.0, seed + 2)
    B = normal_bf16((r, N), 1.0, seed + 3)
    dY = normal_bf16((M, N), 1.0, seed + 4)
    Xd, Ad, Bd, dYd = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    XA = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
    Y = binding.linear_fwd(pk, q, s2, Xd, Ad, Bd, alpha, N, K, XA_out=XA)
    dX, dA, dB = binding.linear_bwd(pk, q, s2, Xd, dYd, Ad, Bd, alpha, N, K, XA=XA)
    dX2, dA2, dB2 = binding.linear_bwd(pk, q, s2, Xd, dYd, Ad, Bd, alpha, N, K, XA=None)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    Xb, Ab, Bb, dYb = map(bf16_bits, (X, A, B, dY))
    Yo, XAo = oracle.linear_fwd(Xb, wq, Ab, Bb, alpha, r)
    dXo, dAo, dBo = oracle.linear_bwd(Xb, dYb, wq, Ab, Bb, alpha, r)
    out = {}
    for name, got, want in (("Y", Y, Yo), ("XA", XA, XAo), ("dX", dX, dXo), ("dA", dA, dAo),
                            ("dB", dB, dBo), ("dX_recompute", dX2, dXo), ("dB_recompute", dB2, dBo)):
        out[name] = (_rel(got, want), _elem(got, want))
        record_property(f"{name}_max_rel", out[name][0])
        record_property(f"{name}_elementwise", out[name][1])
    print(f"M={M} N={N} K={K} r={r}: " + ", ".join(f"{k} {v[0]:.2e}/{v[1]:.2e}" for k, v in out.items()))
    for name, (rel, _) in out.items():
        assert rel <= TOL, f"{name}: max rel error {rel:.3e}"
    return Y, dX


# (M, N, K, r): forward tile / backward tile the library picks on 148 SMs
SHAPES = [
    (1, 1024, 2048, 64),     # few-token stream, one token            | bwd 32-token tiles, split K
    (4, 1024, 512, 8),       # few-token stream, r = 8                | bwd 32-token tiles, split K
    (16, 2048, 1024, 256),   # few-token stream, r = 256              | bwd 32-token tiles, split K
    (24, 1024, 2048, 128),   # 32-token tiles, split K, r = 128       | same
    (300, 512, 1024, 64),    # 256-token tiles + tail, split K        | same
    (2048, 4096, 256, 64),   # 256-token tiles, 256 tiles: no split   | split K
    (2048, 256, 4096, 128),  # 256-token tiles, split K               | 256 tiles: no split
    (512, 1024, 1024, 256),  # r = 256 (four low-rank K blocks)       | same
]


@pytest.mark.parametrize("M,N,K,r", SHAPES)
def test_adapter_term_alone_with_zero_weight(M, N, K, r, record_property):
    Y, dX = _run(M, N, K, r, _zero_weight, 7 * M + N + K + r, record_property)
    # the base product contributes nothing, so a dropped low-rank step would leave zeros
    assert torch.count_nonzero(Y).item() > Y.numel() // 2
    assert torch.count_nonzero(dX).item() > dX.numel() // 2


@pytest.mark.parametrize("M,N,K,r", [(16, 2048, 1024, 64), (24, 1024, 2048, 8), (300, 512, 1024, 64),
                                     (2048, 256, 4096, 128)])
def test_adapter_term_dominant_with_nf4_weight(M, N, K, r, record_property):
    _run(M, N, K, r, _nf4_weight, 11 * M + N + K + r, record_property)


def test_adapter_scale_is_alpha_over_r(record_property):
    """Two alphas on the same W' == 0 layer: Y scales by their ratio up to the
    bf16 rounding of s X A (a swapped or missing scale fails this)."""
    M, N, K, r = 64, 512, 512, 16
    pk, q, s2, _ = _zero_weight(N, K, 5)
    X, A, B = (normal_bf16(s, 1.0, 6 + i).cuda() for i, s in enumerate(((M, K), (K, r), (r, N))))
    Y1 = binding.linear_fwd(pk, q, s2, X, A, B, 16.0, N, K)
    Y2 = binding.linear_fwd(pk, q, s2, X, A, B, 4.0, N, K)  # s = 0.25 vs 1.0: a power of two
    torch.cuda.synchronize()
    # s is a power of two in both calls, so bf16(s XA) scales exactly and so does Y
    assert torch.equal(Y1.float(), (Y2.float() * 4.0))
