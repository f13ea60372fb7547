"""GPU test of qlora_linear_fwd_noalloc, the forward for callers that cannot
allocate device memory (a plugin inside a framework that owns every device
allocation, or a loop that must never enter the allocator).

The entry point takes no workspace: it runs the forward on the library's
fixed device scratch array. It launches the same deterministic kernels as
the ordinary qlora_linear_fwd (caller workspace), so its outputs must be
bit-identical to that call's, on two calls in a row. The two calls use
different inputs, with adapters at N(0, 1) so that the adapter term is
most of Y: the scratch keeps the previous call's contents (among them the
scaled X A operand), and anything that leaked from the first call into the
second would change bits. A shape whose scratch would exceed the fixed
size must be refused.

Named test_zz_* so that pytest collects it last.
"""
import pytest
import torch

from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import normal_bf16, weight_bf16

pytestmark = pytest.mark.gpu


def _layer(M, N, K, r, seed):
    W = weight_bf16(N, K, 0.02, seed, 0.001).cuda()
    pk, am = binding.quantize_nf4(W)
    q, s2 = binding.double_quant(am)
    X = normal_bf16((M, K), 1.0, seed + 1).cuda()
    A = normal_bf16((K, r), 1.0, seed + 2).cuda()
    B = normal_bf16((r, N), 1.0, seed + 3).cuda()
    return pk, q, s2, X, A, B


@pytest.mark.parametrize("M,N,K,r", [(16, 1024, 1024, 8), (40, 256, 192, 16), (4, 2048, 2048, 64),
                                     (2048, 4096, 1024, 64)])
def test_noalloc_matches_workspace_forward_two_calls(M, N, K, r):
    for call, seed in enumerate((11, 23)):
        pk, q, s2, X, A, B = _layer(M, N, K, r, seed + M + N)
        Y_ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        XA_ref = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        binding.linear_fwd(pk, q, s2, X, A, B, 16.0, N, K, Y=Y_ref, XA_out=XA_ref)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        XA = torch.empty((M, r), dtype=torch.bfloat16, device="cuda")
        binding.linear_fwd_noalloc(pk, q, s2, X, A, B, 16.0, N, K, Y=Y, XA_out=XA)
        torch.cuda.synchronize()
        assert binding.device_error() == 0
        assert torch.equal(Y, Y_ref), f"call {call}: Y differs from the workspace forward"
        assert torch.equal(XA, XA_ref), f"call {call}: XA differs from the workspace forward"


def test_noalloc_refuses_oversized_scratch():
    # the forward scratch holds (alpha/r) X A in bf16: 16384 x 256 x 2 bytes = 8 MiB alone
    M, N, K, r = 16384, 1024, 1024, 256
    assert M * r * 2 >= binding.NOALLOC_SCRATCH_BYTES
    pk = torch.empty(N * K // 2, dtype=torch.uint8, device="cuda")
    q = torch.empty(N * K // 64, dtype=torch.uint8, device="cuda")
    s2 = torch.empty((N * K // 64 + 255) // 256, dtype=torch.float32, device="cuda")
    X = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    A = torch.empty((K, r), dtype=torch.bfloat16, device="cuda")
    B = torch.empty((r, N), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(binding.QLoRAError) as ei:
        binding.linear_fwd_noalloc(pk, q, s2, X, A, B, 16.0, N, K)
    assert ei.value.status == 7  # QLORA_ERR_WORKSPACE
