"""The one-pass quantize + double quantization (qlora_quantize_dq; intvml.com
"DL0087 QLoRA", components (2) and (3)) against the oracle's quantize and
double quantization, bit for bit: ragged shapes whose last second-level
group is partial and whose groups straddle rows, non-finite and all-zero
blocks, every pairing of a 4-bit table and an 8-bit map (so both the
bucketed and the binary-search encodes of each level run), with and
without the fp32 block constants written out."""
import itertools

import numpy as np
import pytest
import torch

import oracle
from oracle import codebooks as cb
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, weight_bf16

pytestmark = pytest.mark.gpu


def _check(W, lv=None, t8=None, with_absmax=True):
    N, K = W.shape
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W), lv)
    q_o, s2_o = oracle.double_quant(am_o, t8)
    am = torch.empty(N * K // 64, dtype=torch.float32, device="cuda") if with_absmax else None
    pk, q, s2 = binding.quantize_dq(W.cuda(), nf4=lv, t8=t8, absmax=am)
    torch.cuda.synchronize()
    assert np.array_equal(pk.cpu().numpy(), pk_o)
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_o.view(np.uint32))
    if with_absmax:
        assert np.array_equal(am.cpu().numpy().view(np.uint32), am_o.view(np.uint32))


@pytest.mark.parametrize("N,K", [(1, 64), (3, 192), (192, 1600), (700, 448), (4096, 4096), (333, 11008)])
def test_matches_the_two_oracle_steps(N, K):
    _check(weight_bf16(N, K, 0.02, N + K, 0.001), with_absmax=(N % 2 == 1))


def test_special_blocks():
    N, K = 64, 1024
    W = weight_bf16(N, K, 0.02, 5)
    W[0, :64] = 0.0                         # an all-zero block
    W[1, 5] = float("nan")                  # a NaN weight
    W[2, 70] = float("inf")                 # an infinite weight
    W[3, :] = 0.0                           # zero blocks across a whole row
    W[40:44, :] = 1e-38                     # subnormal-range constants
    W[50, 3] = 3e38                         # a huge constant
    _check(W)


@pytest.mark.parametrize("t4,t8", list(itertools.product(["nf4", "int4", "fp4"], ["linear", "signed", "dynamic"])))
def test_alternative_tables(t4, t8):
    lv = {"nf4": None, "int4": cb.int4_levels(), "fp4": cb.fp4_levels()}[t4]
    tt = {"linear": None, "signed": cb.dq_signed_levels(), "dynamic": cb.dq_dynamic_levels()}[t8]
    _check(weight_bf16(192, 1600, 0.02, 31, 0.002), lv, tt)
