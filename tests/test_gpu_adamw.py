"""GPU parity of the paged AdamW for the adapters (intvml.com "DL0087
QLoRA", component (5) "Paged Optimizers") against the float64 oracle
(oracle/adamw.py: AdamW with decoupled weight decay, Loshchilov and Hutter
2019, Algorithm 2):

* several steps over ragged tensors (1, 1000 and 70 001 elements) in bf16
  and fp16: the fp32 master copy and the moments against the oracle started
  from the same 16-bit parameters and fed the same 16-bit gradients, and the
  16-bit parameters equal to the master rounded to nearest even;
* the state paged out to host memory (a reserve larger than the device's
  free memory stands in for a memory spike): the run completes, the state
  reports its host placement, and every result is bit-identical to the
  device-resident run;
* more tensors than one launch takes (40 segments).
"""
import numpy as np
import pytest
import torch

import oracle
from oracle.adamw import adamw_step
from bit_quantized_lora_blockwise_b200 import binding

pytestmark = pytest.mark.gpu
HYPER = dict(lr=1e-2, betas=(0.9, 0.99), eps=1e-8, weight_decay=0.05)


def _tensors(sizes, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    return [(torch.randn(n, generator=g) * 0.05).to(dtype) for n in sizes]


def _grads(sizes, dtype, seed, steps):
    g = torch.Generator().manual_seed(seed)
    return [[(torch.randn(n, generator=g) * 1e-2).to(dtype) for n in sizes] for _ in range(steps)]


def _run(sizes, dtype, steps, reserve=None):
    params = [p.cuda() for p in _tensors(sizes, dtype, 1)]
    grads = _grads(sizes, dtype, 2, steps)
    opt = binding.PagedAdamW(params, **HYPER)
    if reserve is not None:
        opt.set_reserve(reserve)
    for t in range(steps):
        opt.step([g.cuda() for g in grads[t]])
    torch.cuda.synchronize()
    master, m, v = opt.state()
    out = ([p.cpu() for p in params], master, m, v, opt.location)
    opt.close()
    return out


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_steps_match_oracle(dtype):
    sizes, steps = [1, 1000, 70001], 5
    params, master, m, v, where = _run(sizes, dtype, steps)
    assert where == "device"
    assert binding.device_error() == 0
    p = np.concatenate([t.float().numpy().astype(np.float64) for t in _tensors(sizes, dtype, 1)])
    mo, vo = np.zeros_like(p), np.zeros_like(p)
    for t, gs in enumerate(_grads(sizes, dtype, 2, steps), start=1):
        g = np.concatenate([x.float().numpy().astype(np.float64) for x in gs])
        p, mo, vo = adamw_step(p, mo, vo, g, t, HYPER["lr"], *HYPER["betas"], HYPER["eps"], HYPER["weight_decay"])
    # fp32 state against the float64 oracle: each step moves p by about lr
    assert np.max(np.abs(master - p)) <= 2e-6
    # m cancels where gradients change sign: its error is fp32 rounding of
    # terms of size (1 - b1) |g| (about 1e-3 here), not of m itself
    np.testing.assert_allclose(m, mo, rtol=2e-5, atol=2e-6 * np.max(np.abs(mo)))
    np.testing.assert_allclose(v, vo, rtol=2e-5, atol=1e-16)
    # the 16-bit parameters are the master copy rounded to nearest even
    to16 = oracle.f32_to_bf16 if dtype == torch.bfloat16 else oracle.f32_to_f16
    got = np.concatenate([_bits(t) for t in params])
    assert np.array_equal(got, to16(master))


def test_paged_out_state_gives_identical_results():
    sizes, steps = [4096, 333, 65536], 4
    dev = _run(sizes, torch.bfloat16, steps)
    host = _run(sizes, torch.bfloat16, steps, reserve=1 << 62)  # more than any free memory: a spike
    assert dev[4] == "device" and host[4] == "host"
    assert binding.device_error() == 0
    for a, b in zip(dev[0], host[0]):
        assert torch.equal(a, b)
    for a, b in zip(dev[1:4], host[1:4]):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_more_segments_than_one_launch():
    sizes = [17 * (i + 1) for i in range(40)]
    params, master, m, v, _ = _run(sizes, torch.float16, 2)
    got = np.concatenate([_bits(t) for t in params])
    assert np.array_equal(got, oracle.f32_to_f16(master))
    assert np.all(v > 0)
