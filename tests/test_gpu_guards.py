"""Canary guard bands around every output buffer (the out-of-bounds write
check used in place of a memory sanitizer).

Each output tensor of each call is placed inside a larger device buffer
whose bytes before and after it (guard bands of 4 KB) hold a fixed pattern;
after the call the bands must be unchanged. Shapes are ragged on purpose:
token counts that leave partial 32- and 256-token tiles, weights whose row
count is not a multiple of 128 or 256, K with an odd number of 64-blocks,
second-level groups that end mid-row, and every path of the layer (the
few-token stream, 32-token tiles, CTA pairs with one and two sub-tiles,
split K). Inputs are checked too: the calls must not write them.
"""
import numpy as np
import pytest
import torch

from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import normal_bf16, weight_bf16

pytestmark = pytest.mark.gpu
GUARD = 4096  # bytes on each side (a multiple of 16: keeps the tensor 16-byte aligned)
PATTERN = 0xA5


class Guarded:
    """A tensor of `shape`/`dtype` inside a byte buffer with guard bands."""

    def __init__(self, shape, dtype):
        n = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        self.raw = torch.full((GUARD + n + GUARD,), PATTERN, dtype=torch.uint8, device="cuda")
        self.t = self.raw[GUARD:GUARD + n].view(dtype).view(*shape)

    def intact(self) -> bool:
        head = self.raw[:GUARD]
        tail = self.raw[-GUARD:]
        return bool(torch.all(head == PATTERN).item() and torch.all(tail == PATTERN).item())


def _guarded_copy(x: torch.Tensor) -> Guarded:
    g = Guarded(tuple(x.shape), x.dtype)
    g.t.copy_(x)
    return g


@pytest.mark.parametrize("N,K", [(192, 320), (320, 1600), (64, 64)])
def test_codec_outputs_stay_in_bounds(N, K):
    W = _guarded_copy(weight_bf16(N, K, 0.02, 3, 0.01).cuda())
    nb = N * K // 64
    pk, am = Guarded((N * K // 2,), torch.uint8), Guarded((nb,), torch.float32)
    q, s2 = Guarded((nb,), torch.uint8), Guarded(((nb + 255) // 256,), torch.float32)
    wq = Guarded((N, K), torch.bfloat16)
    w_before = W.t.clone()
    binding.quantize_nf4(W.t, packed=pk.t, absmax=am.t)
    binding.double_quant(am.t, q=q.t, scale2=s2.t)
    binding.dequant(pk.t, q.t, s2.t, N, K, out=wq.t)
    torch.cuda.synchronize()
    for name, g in (("W", W), ("packed", pk), ("absmax", am), ("q", q), ("scale2", s2), ("W'", wq)):
        assert g.intact(), f"{name}: guard band overwritten"
    assert torch.equal(W.t, w_before)


# (M, N, K, r): few-token stream, 32-token tiles, one- and two-sub-tile pairs (split K and not)
@pytest.mark.parametrize("M,N,K,r", [(3, 192, 320, 8), (16, 320, 1600, 16), (24, 192, 448, 64),
                                     (300, 320, 640, 32), (1300, 192, 576, 64), (2048, 4160, 256, 16)])
def test_layer_outputs_stay_in_bounds(M, N, K, r):
    W = weight_bf16(N, K, 0.02, 5, 0.001).cuda()
    pk, am = binding.quantize_nf4(W)
    q, s2 = binding.double_quant(am)
    X = _guarded_copy(normal_bf16((M, K), 1.0, 6).cuda())
    A = _guarded_copy(normal_bf16((K, r), 0.05, 7).cuda())
    B = _guarded_copy(normal_bf16((r, N), 0.05, 8).cuda())
    dY = _guarded_copy(normal_bf16((M, N), 1.0, 9).cuda())
    ins = [(g, g.t.clone()) for g in (X, A, B, dY)]
    Y, XA = Guarded((M, N), torch.bfloat16), Guarded((M, r), torch.bfloat16)
    dX, dA, dB = Guarded((M, K), torch.bfloat16), Guarded((K, r), torch.bfloat16), Guarded((r, N), torch.bfloat16)
    ws = Guarded((binding.workspace_bytes(M, N, K, r),), torch.uint8)
    binding.linear_fwd(pk, q, s2, X.t, A.t, B.t, 16.0, N, K, Y=Y.t, XA_out=XA.t, workspace=ws.t)
    binding.linear_bwd(pk, q, s2, X.t, dY.t, A.t, B.t, 16.0, N, K, XA=XA.t, dX=dX.t, dA=dA.t, dB=dB.t,
                       workspace=ws.t)
    binding.linear_bwd(pk, q, s2, X.t, dY.t, A.t, B.t, 16.0, N, K, XA=None, dX=dX.t, dA=dA.t, dB=dB.t,
                       workspace=ws.t)
    Y2 = Guarded((M, N), torch.bfloat16)
    binding.linear_fwd_noalloc(pk, q, s2, X.t, A.t, B.t, 16.0, N, K, Y=Y2.t)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    for name, g in (("Y", Y), ("XA", XA), ("dX", dX), ("dA", dA), ("dB", dB), ("workspace", ws),
                    ("Y (no-alloc)", Y2)):
        assert g.intact(), f"{name}: guard band overwritten"
    for g, before in ins:
        assert g.intact() and torch.equal(g.t, before), "an input was written"
    assert torch.equal(Y.t, Y2.t)
