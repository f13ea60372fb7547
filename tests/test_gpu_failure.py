"""Failure detection on the GPU without a fault. Every device-side wait in the
library is bounded, and the library's allocations can be made to fail on
the host. The self-test kernel waits on an mbarrier phase that
nothing completes; the wait must give up after its limit, report through
bit 0 of the device error word, and leave the context usable (a forward right
after it matches the oracle and reports no error)."""
import threading

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


# --- host-side allocation fault injection -----------------------------------
# The paged optimizers exist so that a memory spike does not end the run
# (promptingindex.com "QLoRA: Finetuning 65B Models on a Single GPU", "Double
# Quantization and Paged Optimizers"). Here the library's own allocations are
# made to fail on the host, without touching the GPU: each failing call must
# return QLORA_ERR_CUDA, launch nothing, leave no half-built state, and the
# same call must then succeed with the results of an undisturbed run.

@pytest.fixture(autouse=True)
def _no_pending_injection():
    """No injected allocation failure outlives the test that set it."""
    yield
    binding.debug_fail_allocs(0)


def _adapter_params(seed):
    shapes = ((256, 16), (16, 512), (320, 8))
    params = [normal_bf16(s, 0.05, seed + i).cuda() for i, s in enumerate(shapes)]
    grads = [normal_bf16(s, 1e-2, seed + 10 + i).cuda() for i, s in enumerate(shapes)]
    return params, grads


def test_paged_adamw_create_fails_then_recovers(cuda_device):
    params, grads = _adapter_params(40)
    ref = [p.clone() for p in params]
    binding.debug_fail_allocs(0)
    launches = binding.launch_count()
    binding.debug_fail_allocs(1)
    with pytest.raises(binding.QLoRAError) as err:
        binding.PagedAdamW(params)
    assert err.value.status == 5  # QLORA_ERR_CUDA
    assert binding.debug_fail_allocs(0) == 0, "the failure was consumed"
    assert binding.launch_count() == launches, "a failed create launches nothing"
    assert all(torch.equal(p, q) for p, q in zip(params, ref)), "parameters untouched"

    opt, base = binding.PagedAdamW(params, lr=1e-3), binding.PagedAdamW(ref, lr=1e-3)
    for _ in range(2):
        opt.step(grads)
        base.step(grads)
    torch.cuda.synchronize()
    assert all(torch.equal(p, q) for p, q in zip(params, ref))
    opt.close()
    base.close()


def _two_linears(M, r, seed):
    out = []
    for i, (N, K) in enumerate(((512, 256), (256, 512))):
        W = weight_bf16(N, K, 0.02, seed + 10 * i)
        pk, am = binding.quantize_nf4(W.cuda())
        q, s2 = binding.double_quant(am)
        out.append({"packed": pk, "q": q, "scale2": s2, "N": N, "K": K,
                    "X": normal_bf16((M, K), 1.0, seed + 10 * i + 1).cuda(),
                    "A": normal_bf16((K, r), 0.05, seed + 10 * i + 2).cuda(),
                    "B": normal_bf16((r, N), 0.05, seed + 10 * i + 3).cuda(),
                    "Y": torch.empty((M, N), dtype=torch.bfloat16, device="cuda"),
                    "XA": torch.empty((M, r), dtype=torch.bfloat16, device="cuda")})
    return out


@pytest.mark.parametrize("skip", [0, 1, 2])
def test_block_stream_setup_fails_then_recovers(cuda_device, skip):
    """The block executor's per-thread streams and events are made on a
    thread's first block call (fork event, side stream, join event). Failing
    the first, second or third of them must free the ones already made and
    leave the thread able to set them up on its next call."""
    M, r = 40, 16
    lins = _two_linears(M, r, 60)
    binding.block_fwd(lins, M, r, 16.0)  # this thread's streams: the undisturbed run
    torch.cuda.synchronize()
    want = [(L["Y"].clone(), L["XA"].clone()) for L in lins]
    for L in lins:
        L["Y"].zero_()
        L["XA"].zero_()

    result = {}

    def fresh_thread():  # a new host thread has no streams yet
        try:
            launches = binding.launch_count()
            binding.debug_fail_allocs(1, skip=skip)
            try:
                binding.block_fwd(lins, M, r, 16.0)
                result["first"] = 0
            except binding.QLoRAError as e:
                result["first"] = e.status
            result["launched"] = binding.launch_count() - launches
            result["pending"] = binding.debug_fail_allocs(0)
            binding.block_fwd(lins, M, r, 16.0)
            torch.cuda.synchronize()
            result["second"] = 0
        except Exception as e:  # reported to the test thread below
            result["error"] = repr(e)

    t = threading.Thread(target=fresh_thread)
    t.start()
    t.join()
    assert "error" not in result, result.get("error")
    assert result["first"] == 5, "the setup failure is QLORA_ERR_CUDA"
    assert result["launched"] == 0, "the failed call launches nothing"
    assert result["pending"] == 0
    assert result["second"] == 0
    for L, (Y, XA) in zip(lins, want):
        assert torch.equal(L["Y"], Y) and torch.equal(L["XA"], XA)
