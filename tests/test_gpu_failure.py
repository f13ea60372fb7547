"""Failure detection on the GPU without a fault: every device-side wait in the
library is bounded. The self-test kernel waits on an mbarrier phase that
nothing completes; the wait must give up after its limit, report through
bit 0 of the device error word, and leave the context usable (a forward right
after it matches the oracle and reports no error)."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import weight_bf16, normal_bf16, bf16_bits

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_and_context_survives(cuda_device):
    binding.device_error(clear=True)
    binding.selftest_bounded_wait()
    torch.cuda.synchronize()
    assert binding.device_error(clear=True) & 1 == 1, "the wait that cannot complete must report"
    assert binding.device_error() == 0, "clearing resets the word"

    # the device is still fully usable: a small forward is correct
    M, N, K, r = 16, 256, 192, 8
    W = weight_bf16(N, K, 0.02, 7)
    X = normal_bf16((M, K), 1.0, 8)
    A = normal_bf16((K, r), 0.01, 9)
    B = normal_bf16((r, N), 0.01, 10)
    pk, am = binding.quantize_nf4(W.cuda())
    q, s2 = binding.double_quant(am)
    Y = binding.linear_fwd(pk, q, s2, X.cuda(), A.cuda(), B.cuda(), 16.0, N, K)
    torch.cuda.synchronize()
    assert binding.device_error() == 0
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W))
    q_o, s2_o = oracle.double_quant(am_o)
    Wq = oracle.dequant(pk_o, q_o, s2_o, N * K).reshape(N, K)
    Yo, _ = oracle.linear_fwd(bf16_bits(X), Wq, bf16_bits(A), bf16_bits(B), 16.0, r)
    y = Y.float().cpu().numpy().astype(np.float64)
    assert np.max(np.abs(y - Yo)) / np.max(np.abs(Yo)) <= 1e-2
