"""Pins of the oracle's codec (absmax, NF4 encode, double quant, dequant).

What the pages fix and how each is pinned here:
* blocks of 64 with one absmax each (intvml.com "DL0087 QLoRA", component 2):
  absmax against numpy's own max; buffer sizes;
* nearest-level encoding to a stored 4-bit code (DL0087 formulation list):
  the midpoint counting rule against a brute-force argmin of distances over
  every bf16 bit pattern in [-1, 1];
* double quantization, 8-bit codes with one fp32 scale per 256 constants
  (DL0087 component 3; promptingindex.com "Double Quantization"): group
  maxima against numpy, error of the linear 8-bit code <= S/510, groups that
  straddle rows;
* dequantization feeding the matmul (DL0087 opening paragraph): closed-form
  values (zero code -> 0, extreme codes -> +-S), and the round-trip bound
  |w - w'| <= (gap/2) c + |c - c'| + bf16 rounding;
* storage: 4 + 8/64 + 32/(64*256) bits per parameter and the page figures in
  tests/golden/page_figures.json (7B: 14 GB -> 3.6 GB; 65B DQ saving ~3 GB).
"""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))


def _bf16_bits_of(x):
    """numpy float32 -> bf16 bits by round-to-nearest-even (test's own helper,
    written with numpy integer ops, independent of the oracle's C helper)."""
    u = np.asarray(x, np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)


def _f32_of_bits(b):
    return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _rand_w(n, k, seed, std=0.02, outliers=0.0):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal(n * k) * std).astype(np.float32)
    if outliers:
        pos = rng.integers(0, n * k, int(outliers * n * k))
        w[pos] = np.sign(rng.standard_normal(pos.size)) * 10 * std
    return _bf16_bits_of(w).reshape(n, k)


def test_absmax_matches_numpy():
    w = _rand_w(8, 256, 1, outliers=0.01)
    got = oracle.absmax(w)
    want = np.abs(_f32_of_bits(w)).reshape(-1, 64).max(axis=1)
    assert got.shape == (8 * 256 // 64,)
    assert np.array_equal(got, want)


def test_nearest_level_bruteforce_exhaustive_bf16():
    """Every finite bf16 x with |x| <= 1, encoded with absmax 1 (so x = w)."""
    L = oracle.nf4_levels()
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    x = _f32_of_bits(bits)
    keep = np.isfinite(x) & (np.abs(x) <= 1.0)
    bits, x = bits[keep], x[keep]
    pad = (-bits.size) % 64
    w = np.concatenate([bits, np.zeros(pad, np.uint16)])
    amax = np.ones(w.size // 64, np.float32)
    packed = oracle.encode_nf4(w, amax, L)
    codes = np.empty(w.size, np.int64)
    codes[0::2] = packed & 0x0F
    codes[1::2] = packed >> 4
    codes = codes[:x.size]
    d = np.abs(x.astype(np.float64)[:, None] - L.astype(np.float64)[None, :])
    brute = d.argmin(axis=1)  # first minimum = lower level on exact ties
    srt = np.sort(d, axis=1)
    clear = (srt[:, 1] - srt[:, 0]) > 1e-6
    assert clear.sum() == x.size  # no bf16 value sits on an NF4 midpoint
    assert x.size > 32000
    assert np.array_equal(codes[clear], brute[clear])
    for i in range(15):
        m = np.float32((L[i] + L[i + 1]) * np.float32(0.5))
        assert oracle.nearest_level(float(m), L) == i
        assert oracle.nearest_level(float(np.nextafter(m, np.float32(2))), L) == i + 1


def test_nibble_order_and_codes_of_exact_levels():
    L = oracle.nf4_levels()
    codes = np.array([(3 * e + 5) % 16 for e in range(64)])
    w = _bf16_bits_of(L[codes] * np.float32(0.5))  # absmax becomes 0.5 (codes 0 and 15 present)
    assert {0, 15} <= set(codes.tolist())
    packed, amax = oracle.quantize_nf4(w)
    assert amax.tolist() == [0.5]
    expect = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    assert np.array_equal(packed, expect)


def test_zero_block_and_zero_group():
    w = np.zeros((1, 128), np.uint16)
    w[0, 64:] = _rand_w(1, 64, 3)
    packed, amax = oracle.quantize_nf4(w)
    assert amax[0] == 0.0
    assert np.all(packed[:32] == 0x77)  # code 7 is the exact zero level
    q, s2 = oracle.double_quant(np.zeros(10, np.float32))
    assert np.all(q == 0) and s2.tolist() == [0.0]
    out = oracle.dequant(packed, *oracle.double_quant(amax), 128)
    assert np.all(_f32_of_bits(out[:64]) == 0.0)


def test_double_quant_groups_straddle_rows_and_partial_tail():
    # K = 5120 -> 80 blocks per row; 256-constant groups straddle rows
    w = _rand_w(7, 5120, 4, outliers=0.001)
    _, amax = oracle.quantize_nf4(w)
    nb = amax.size
    assert nb == 7 * 80 and nb % 256 != 0
    q, s2 = oracle.double_quant(amax)
    assert s2.size == -(-nb // 256)
    for g in range(s2.size):
        assert s2[g] == amax[256 * g: 256 * (g + 1)].max()
    cprime = oracle.dq_constants(q, s2)
    S = np.repeat(s2, 256)[:nb]
    err = np.abs(cprime.astype(np.float64) - amax)
    assert np.all(err <= S / 510.0 * (1 + 1e-6) + S * 2.0 ** -23)
    # the group maximum itself is carried exactly (code 255 -> T8 = 1)
    for g in range(s2.size):
        j = 256 * g + int(np.argmax(amax[256 * g: 256 * (g + 1)]))
        assert q[j] == 255 and cprime[j] == s2[g]


def test_dequant_closed_forms():
    L = oracle.nf4_levels()
    # one block whose codes run 0..15 four times; one group with S = 3
    codes = np.tile(np.arange(16), 4)
    packed = (codes[0::2] | (codes[1::2] << 4)).astype(np.uint8)
    out = _f32_of_bits(oracle.dequant(packed, np.array([255], np.uint8),
                                      np.array([3.0], np.float32), 64))
    assert out[7] == 0.0                       # exact zero level
    assert out[15] == 3.0 and out[0] == -3.0   # +-S at the extremes (L = +-1, T8[255] = 1)
    # q = 0 -> c' = 0 -> every weight 0
    out0 = _f32_of_bits(oracle.dequant(packed, np.array([0], np.uint8),
                                       np.array([3.0], np.float32), 64))
    assert np.all(out0 == 0.0)
    # a power-of-two c' scales exactly: bf16(2 L_i) == 2 bf16(L_i)
    out2 = _f32_of_bits(oracle.dequant(packed, np.array([255], np.uint8),
                                       np.array([2.0], np.float32), 64))
    assert np.array_equal(out2[:16], 2 * _f32_of_bits(_bf16_bits_of(L)))


def test_roundtrip_error_bound():
    """|w - w'| <= (gap/2 + 2^-24) c + |c - c'| + 2^-8 |w'| + 2^-24 |w'|,
    gap = width of the level interval holding x = w / c."""
    L = oracle.nf4_levels().astype(np.float64)
    n, k = 64, 1024
    w = _rand_w(n, k, 5, outliers=0.001)
    packed, amax = oracle.quantize_nf4(w)
    q, s2 = oracle.double_quant(amax)
    wq = _f32_of_bits(oracle.dequant(packed, q, s2, n * k)).astype(np.float64)
    wf = _f32_of_bits(w).astype(np.float64).reshape(-1)
    c = np.repeat(amax.astype(np.float64), 64)
    cp = np.repeat(oracle.dq_constants(q, s2).astype(np.float64), 64)
    x = np.where(c > 0, wf / np.where(c > 0, c, 1), 0)
    idx = np.clip(np.searchsorted(L, x, side="right") - 1, 0, 14)
    gap = L[idx + 1] - L[idx]
    bound = (gap / 2 + 2.0 ** -24) * c + np.abs(c - cp) + (2.0 ** -8 + 2.0 ** -24) * np.abs(wq)
    assert np.all(np.abs(wf - wq) <= bound * (1 + 1e-9))


def test_storage_matches_page_figures():
    n, k = 64, 4096  # n*k % (64*256) == 0
    w = _rand_w(n, k, 6)
    packed, amax = oracle.quantize_nf4(w)
    q, s2 = oracle.double_quant(amax)
    bits = 8.0 * (packed.nbytes + q.nbytes + s2.nbytes) / (n * k)
    assert bits == 4.126953125  # 4 + 8/64 + 32/(64*256), exactly
    assert amax.size == n * k // GOLDEN["block_size"]["value"]
    assert s2.size == amax.size // GOLDEN["dq_block_size"]["value"]
    payload = 8.0 * packed.nbytes / (n * k)
    first = 8.0 * q.nbytes / (n * k)
    second = 8.0 * s2.nbytes / (n * k)
    assert payload == GOLDEN["bits_payload"]["value"]
    assert first == GOLDEN["bits_first_level_constants"]["value"]
    assert abs(second - GOLDEN["bits_second_level_scales"]["value"]) <= 0.001
    before = 32.0 / 64  # fp32 absmax per 64 weights, no DQ
    assert before == GOLDEN["metadata_bits_before_dq"]["value"]
    assert abs((first + second) - GOLDEN["metadata_bits_after_dq"]["value"]) <= 0.001
    saving = before - (first + second)
    assert abs(saving - GOLDEN["dq_saving_bits_per_param"]["value"]) <= 0.01
    g = GOLDEN["dq_saving_65b_gb"]
    assert abs(saving * g["params"] / 8 / 1e9 - g["value"]) <= g["rounded_to"]
    g = GOLDEN["frozen_7b_qlora_gb"]
    assert abs(bits * g["params"] / 8 / 1e9 - g["value"]) <= g["rounded_to"]
    g = GOLDEN["frozen_7b_bf16_gb"]
    assert abs(16 * g["params"] / 8 / 1e9 - g["value"]) <= g["rounded_to"]
    assert 16 * GOLDEN["storage_70b_16bit_gb"]["params"] / 8 / 1e9 == GOLDEN["storage_70b_16bit_gb"]["value"]
    assert payload * GOLDEN["storage_70b_4bit_gb"]["params"] / 8 / 1e9 == GOLDEN["storage_70b_4bit_gb"]["value"]


def test_bf16_conversions_match_torch():
    """The oracle's fp32 <-> bf16 helpers against torch's conversions (an
    independent library routine): widening is exact, narrowing rounds to
    nearest even, on ties (low half 0x8000), neighbours of ties, subnormals,
    infinities and the largest finite values."""
    import torch
    rng = np.random.default_rng(7)
    hi = rng.integers(0, 1 << 16, 4096, dtype=np.uint32)
    lows = np.array([0x0000, 0x0001, 0x7FFF, 0x8000, 0x8001, 0xFFFF], np.uint32)
    bits = (hi[:, None] << 16 | lows[None, :]).reshape(-1)
    bits = np.concatenate([bits, np.array([0x7F7FFFFF, 0xFF7FFFFF, 0x7F800000, 0xFF800000, 0x00000001,
                                           0x807FFFFF, 0x00008000, 0x7F7F8000], np.uint32)])
    x = bits.view(np.float32)
    finite_or_inf = ~np.isnan(x)
    x = x[finite_or_inf]
    got = oracle.f32_to_bf16(x)
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)
    back = oracle.bf16_to_f32(got)
    want_back = torch.from_numpy(want.view(np.int16).copy()).view(torch.bfloat16).float().numpy()
    assert np.array_equal(back.view(np.uint32), want_back.view(np.uint32))
