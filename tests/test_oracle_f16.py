"""Pins of the oracle's fp16 path (the pages' other 16-bit compute type:
systemoverflow.com "QLoRA: Efficient Finetuning of Quantized LLMs at Extreme
Scale" runs the adapters and the computation in 16-bit float or bfloat16).

The oracle's binary32 -> binary16 conversion is written from the IEEE 754
format on bit patterns; it is checked here against numpy's own float32 ->
float16 cast (a correctly rounded, round-to-nearest-even library routine
that shares nothing with it) over every exponent the conversion
distinguishes, with the rounding ties, the overflow threshold and the
subnormal range spelled out. The fp16 dequantization is then checked
against the definition evaluated with numpy: L[code] * c' in float32, then
cast to float16.
"""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _numpy_f16_bits(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, np.float32).astype(np.float16).view(np.uint16)


def _from_bits(u) -> np.ndarray:
    return np.asarray(u, np.uint32).view(np.float32)


def test_conversion_matches_numpy_over_every_exponent():
    rng = np.random.default_rng(0)
    vals = []
    # every binary32 exponent from far below the fp16 subnormals to past inf
    for E in range(80, 256):
        frac = rng.integers(0, 1 << 23, 512, dtype=np.uint32)
        # the fraction bits below each rounding position: exact ties, one
        # below and one above, for every shift the subnormal path uses
        for sh in range(12, 25):
            t = np.uint32(1 << (sh - 1)) if sh - 1 < 23 else np.uint32(0)
            base = rng.integers(0, 1 << 23, 4, dtype=np.uint32) & ~np.uint32((1 << min(sh, 23)) - 1)
            frac = np.concatenate([frac, base | t, (base | t) - 1, (base | t) + 1])
        frac &= np.uint32(0x7FFFFF)
        u = (np.uint32(E) << np.uint32(23)) | frac
        vals.append(u)
        vals.append(u | np.uint32(0x80000000))
    u = np.concatenate(vals)
    x = _from_bits(u)
    finite = ~np.isnan(x)
    got = oracle.f32_to_f16(x)
    want = _numpy_f16_bits(x)
    assert np.array_equal(got[finite], want[finite])
    # NaN stays NaN (sign kept)
    assert np.all(np.isnan(got[~finite].view(np.float16)))


@pytest.mark.parametrize("x,bits", [
    (65504.0, 0x7BFF),            # largest finite
    (65519.99609375, 0x7BFF),     # just below the half-way point
    (65520.0, 0x7C00),            # half-way, ties to even (the next "value" is inf)
    (float("inf"), 0x7C00),
    (2.0 ** -14, 0x0400),         # least normal
    (2.0 ** -24, 0x0001),         # least subnormal
    (2.0 ** -25, 0x0000),         # half of it: ties to even (zero)
    (1.5 * 2.0 ** -25, 0x0001),
    (3 * 2.0 ** -25, 0x0002),     # 1.5 units: ties to even (2)
    (-0.0, 0x8000),
    (1.0, 0x3C00),
    (1.0 + 2.0 ** -11, 0x3C00),   # tie below an even fraction
    (1.0 + 3 * 2.0 ** -11, 0x3C02),
])
def test_conversion_spelled_out_cases(x, bits):
    assert int(oracle.f32_to_f16(np.array([x], np.float32))[0]) == bits


def _state(nb, seed, scale_lo, scale_hi):
    rng = np.random.default_rng(seed)
    packed = rng.integers(0, 256, nb * 32, dtype=np.uint8)
    q = rng.integers(0, 256, nb, dtype=np.uint8)
    ng = (nb + 255) // 256
    scale2 = np.exp(rng.uniform(np.log(scale_lo), np.log(scale_hi), ng)).astype(np.float32)
    return packed, q, scale2


@pytest.mark.parametrize("lo,hi", [(1e-3, 1.0), (1e3, 1e6), (1e-9, 1e-5)])
def test_dequant_f16_is_the_definition(lo, hi):
    """W'[e] = f16(L[code] * c') with c' = t8[q] * S in float32: ordinary,
    overflowing (to inf) and subnormal magnitudes."""
    nb = 700  # three second-level groups, the last one partial
    packed, q, scale2 = _state(nb, 7, lo, hi)
    L = oracle.nf4_levels()
    cp = oracle.dq_constants(q, scale2)
    codes = np.empty(nb * 64, np.int64)
    codes[0::2] = packed & 0x0F
    codes[1::2] = packed >> 4
    prod = (L[codes].astype(np.float32) * np.repeat(cp, 64).astype(np.float32)).astype(np.float32)
    want = _numpy_f16_bits(prod)
    got = oracle.dequant_f16(packed, q, scale2, nb * 64)
    assert np.array_equal(got, want)
    if hi > 1e5:
        assert np.any(got == 0x7C00) or np.any(got == 0xFC00)
    if hi < 1e-4:
        assert np.any((got & 0x7C00) == 0) and np.any((got & 0x03FF) != 0)


def test_dequant_f16_and_bf16_share_the_codes():
    """Both roundings of the same fp32 products: where the product is exact
    in both formats (the zero level, and the +-1 levels times a power-of-two
    constant) the two outputs are the same number."""
    nb = 512
    packed = np.full(nb * 32, 0xF0, np.uint8)        # code 0 (-1) then code 15 (+1)
    packed[: nb * 16] = 0x77                           # first half: the zero level
    q = np.full(nb, 255, np.uint8)                     # t8[255] = 1
    scale2 = np.array([2.0 ** -3, 2.0 ** 5], np.float32)
    wb = oracle.dequant(packed, q, scale2, nb * 64)
    wh = oracle.dequant_f16(packed, q, scale2, nb * 64)
    fb = (wb.astype(np.uint32) << 16).view(np.float32)
    fh = wh.view(np.float16).astype(np.float32)
    assert np.array_equal(fb, fh)
    half = nb * 32
    assert np.all(fh[:half] == 0.0)
    assert set(np.unique(fh[half:]).tolist()) == {-32.0, 32.0}
