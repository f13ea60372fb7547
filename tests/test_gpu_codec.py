"""GPU parity of the codec kernels against the CPU oracle, bit-exact.

Quantize (packed nibbles + absmax), double quant (8-bit codes + scales) and
dequant (bf16 weights) are integer/byte results or exact fp32 decisions:
every byte must equal the oracle's. Inputs: seeded synthetic weights with
the workloads' distributions (N(0, 0.02) with 0.1 % outliers at +-10 sigma),
ragged shapes (odd row counts, constants that straddle rows and a short last
group), and an exhaustive sweep of every bf16 weight against every bf16
absmax mantissa, plus tiny and zero blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_lora_blockwise_b200 import binding
from bit_quantized_lora_blockwise_b200.inputs import weight_bf16, bf16_bits

pytestmark = pytest.mark.gpu


def _bits_to_cuda(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).cuda()


def _codec_parity(W_cpu: torch.Tensor):
    N, K = W_cpu.shape
    bits = bf16_bits(W_cpu)
    pk_o, am_o = oracle.quantize_nf4(bits)
    q_o, s2_o = oracle.double_quant(am_o)
    wq_o = oracle.dequant(pk_o, q_o, s2_o, N * K)
    W = W_cpu.cuda()
    pk, am = binding.quantize_nf4(W)
    q, s2 = binding.double_quant(am)
    wq = binding.dequant(pk, q, s2, N, K)
    torch.cuda.synchronize()
    assert np.array_equal(am.cpu().numpy(), am_o), "absmax"
    assert np.array_equal(pk.cpu().numpy(), pk_o), "packed nibbles"
    assert np.array_equal(q.cpu().numpy(), q_o), "8-bit constant codes"
    assert np.array_equal(s2.cpu().numpy(), s2_o), "second-level scales"
    assert np.array_equal(bf16_bits(wq).reshape(-1), wq_o), "dequantized bf16"
    assert binding.device_error() == 0


@pytest.mark.parametrize("N,K,std,outl", [
    (1024, 1024, 0.02, 0.0),      # single-linear workload
    (7, 5120, 0.02, 0.001),       # 560 constants: groups straddle rows, short last group
    (3, 64, 0.02, 0.0),           # one block per row, 3 constants
    (4096, 4096, 0.02, 0.001),    # 7B q/k/v/o shape with outliers
    (257, 11008, 0.015, 0.0),     # 11008 = 172 blocks per row
])
def test_codec_bit_exact(N, K, std, outl):
    W = weight_bf16(N, K, std, seed=1234 + N + K, outlier_frac=outl)
    _codec_parity(W)


def test_codec_exhaustive_ratio_sweep():
    """Every bf16 |w| <= c for every bf16 mantissa of c in [1, 2): the
    quotient w / c then covers every pair of bf16 significands."""
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (allbits.astype(np.uint32) << 16).view(np.float32)
    rows = []
    for m in range(128):
        cbits = np.uint16(0x3F80 + m)                       # c = 1 + m/128
        c = np.float32((np.uint32(cbits) << 16).view(np.float32))
        sel = allbits[np.isfinite(vals) & (np.abs(vals) <= c)]
        pad = (-sel.size) % 63
        sel = np.concatenate([sel, np.zeros(pad, np.uint16)]).reshape(-1, 63)
        blocks = np.concatenate([sel, np.full((sel.shape[0], 1), cbits, np.uint16)], axis=1)
        rows.append(blocks.reshape(-1))
    flat = np.concatenate(rows)
    flat = np.concatenate([flat, np.zeros((-flat.size) % 4096, np.uint16)])
    W = torch.from_numpy(flat.view(np.int16)).view(torch.bfloat16).view(-1, 4096)
    _codec_parity(W)


def test_codec_tiny_and_zero_blocks():
    rng = np.random.default_rng(7)
    K = 256
    rows = []
    # subnormal-only blocks (absmax below 2^-125 goes through the IEEE divide)
    rows.append(rng.integers(0, 0x80, K, dtype=np.uint16) | (rng.integers(0, 2, K, dtype=np.uint16) << 15))
    # blocks around the 2^-125 boundary
    rows.append(rng.integers(0x0080, 0x0140, K, dtype=np.uint16))
    # all-zero row, and -0.0 entries
    rows.append(np.zeros(K, np.uint16))
    rows.append(np.full(K, 0x8000, np.uint16))
    # huge magnitudes
    rows.append(rng.integers(0x7E00, 0x7F7F, K, dtype=np.uint16) | (rng.integers(0, 2, K, dtype=np.uint16) << 15))
    W = torch.from_numpy(np.stack(rows).view(np.int16)).view(torch.bfloat16)
    _codec_parity(W)


def test_custom_tables_are_honoured():
    """A different ascending NF4-style table and 8-bit map pass through."""
    N, K = 64, 512
    W = weight_bf16(N, K, 0.02, seed=99)
    lv = np.array([-1, -.8, -.6, -.45, -.3, -.2, -.1, 0, .05, .1, .2, .3, .45, .6, .8, 1], np.float32)
    t8 = (np.arange(256, dtype=np.float64) / 255.0) ** 2
    t8 = t8.astype(np.float32)
    bits = bf16_bits(W)
    pk_o, am_o = oracle.quantize_nf4(bits, lv)
    q_o, s2_o = oracle.double_quant(am_o, t8)
    wq_o = oracle.dequant(pk_o, q_o, s2_o, N * K, lv, t8)
    Wc = W.cuda()
    pk, am = binding.quantize_nf4(Wc, nf4=lv)
    q, s2 = binding.double_quant(am, t8=t8)
    wq = binding.dequant(pk, q, s2, N, K, nf4=lv, t8=t8)
    assert np.array_equal(pk.cpu().numpy(), pk_o)
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert np.array_equal(bf16_bits(wq).reshape(-1), wq_o)


def _dq_boundary_constants(t8: np.ndarray, rng) -> np.ndarray:
    """Groups of 256 constants whose ratios c / S sit on and next to every
    fp32 midpoint of t8, for several group maxima S, plus degenerate groups."""
    t8 = t8.astype(np.float32)
    mids = ((t8[:-1] + t8[1:]) * np.float32(0.5)).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(2))])
    groups = []
    for S in (np.float32(1.0), np.float32(0.37), np.float32(3.0e-3), np.float32(2.5e4)):
        vals = (near * S).astype(np.float32)
        vals = np.concatenate([vals, np.nextafter(vals, np.float32(0)), np.nextafter(vals, np.float32(np.inf))])
        vals = np.clip(vals, 0, S).astype(np.float32)
        vals = vals[rng.permutation(vals.size)]
        for i in range(0, vals.size, 255):
            g = np.concatenate([[S], vals[i:i + 255]]).astype(np.float32)
            groups.append(np.concatenate([g, np.zeros(256 - g.size, np.float32)]))
    tiny = np.float32(2.0 ** -130)           # subnormal group maximum: IEEE divide path
    groups.append(np.concatenate([[tiny], (rng.random(255) * tiny).astype(np.float32)]))
    big = np.float32(2.0 ** 126)             # group maximum above the reciprocal range
    groups.append(np.concatenate([[big], (rng.random(255) * big).astype(np.float32)]))
    groups.append(np.zeros(256, np.float32))                                  # all zero
    groups.append(np.concatenate([[np.float32(1.0)], -rng.random(255).astype(np.float32)]))  # negatives
    odd = rng.random(256).astype(np.float32)
    odd[3], odd[9], odd[17] = np.nan, -0.0, np.float32(1e-42)
    groups.append(odd)
    inf = rng.random(256).astype(np.float32)
    inf[5] = np.inf
    groups.append(inf)
    return np.concatenate(groups).astype(np.float32)


@pytest.mark.parametrize("table", ["default", "grid256", "shifted"])
def test_double_quant_midpoint_boundaries(table):
    """Every midpoint, its fp32 neighbours, several group scales, negative,
    NaN, infinite, zero and subnormal constants: bit-exact against the
    oracle for tables on the bucketed encode and the binary search."""
    rng = np.random.default_rng(11)
    if table == "default":
        t8 = oracle.dq_levels()
    elif table == "grid256":
        # midpoints (k + 1/2) / 256 fall exactly on bucket edges
        t8 = (np.arange(256, dtype=np.float64) / 256.0).astype(np.float32)
    else:
        t8 = (0.001 + np.arange(256, dtype=np.float64) * (0.999 / 255.0)).astype(np.float32)
    am = _dq_boundary_constants(t8, rng)
    am = np.concatenate([am, rng.random(77).astype(np.float32)])  # short last group
    q_o, s2_o = oracle.double_quant(am, t8)
    q, s2 = binding.double_quant(torch.from_numpy(am).cuda(), t8=t8)
    torch.cuda.synchronize()
    assert np.array_equal(s2.cpu().numpy().view(np.uint32), s2_o.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), q_o)
    assert binding.device_error() == 0


def test_quantize_nonfinite_weights():
    """NaN and infinite weights: the block maximum ignores NaN, a NaN
    quotient (NaN weight, or inf / inf) has no midpoint below it (code 0),
    finite weights of a block with an infinite maximum quantize to zero."""
    rng = np.random.default_rng(5)
    K = 512
    rows = []
    for special in (0x7FC0, 0xFFC0, 0x7F80, 0xFF80):   # +NaN, -NaN, +inf, -inf
        r = weight_bf16(1, K, 0.02, seed=int(special)).view(torch.int16).numpy().view(np.uint16).reshape(-1).copy()
        idx = rng.choice(K, 9, replace=False)
        r[idx] = special
        rows.append(r)
    bits = np.stack(rows)
    pk_o, am_o = oracle.quantize_nf4(bits)
    W = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()
    pk, am = binding.quantize_nf4(W)
    torch.cuda.synchronize()
    assert np.array_equal(am.cpu().numpy().view(np.uint32), am_o.view(np.uint32)), "absmax"
    assert np.array_equal(pk.cpu().numpy(), pk_o), "packed nibbles"
    assert binding.device_error() == 0


def test_quantize_input_only_16_byte_aligned():
    """A weight that starts 16 bytes into an allocation (16- but not
    32-byte aligned) takes the 16-byte load path; results are identical."""
    N, K = 96, 1024
    W = weight_bf16(N, K, 0.02, seed=3, outlier_frac=0.001)
    buf = torch.zeros(N * K + 64, dtype=torch.bfloat16, device="cuda")
    Wv = buf[8:8 + N * K].view(N, K)
    Wv.copy_(W.cuda())
    assert Wv.data_ptr() % 32 == 16
    pk_o, am_o = oracle.quantize_nf4(bf16_bits(W))
    pk, am = binding.quantize_nf4(Wv)
    torch.cuda.synchronize()
    assert np.array_equal(am.cpu().numpy(), am_o)
    assert np.array_equal(pk.cpu().numpy(), pk_o)
