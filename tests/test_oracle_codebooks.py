"""Pins of the oracle's alternative code tables and of the comparison the
pages make with them (promptingindex.com "Finetuning 65B Models on a Single
GPU", section "4-bit NormalFloat": the 4-bit NormalFloat type outperforms
4-bit integers and 4-bit floats; intvml.com "DL0087 QLoRA", component 1).

* INT4: the codec's midpoint rule on the levels i / 7 must give the code of
  plain absmax rounding, round(7 x), for every x that is not a tie.
* FP4: the levels must be the values of the E2M1 format, decoded here from
  its bit layout (sign bit, two exponent bits with bias 1, one mantissa
  bit; exponent 0 is subnormal), over its largest value.
* the 8-bit maps: endpoints, symmetry / octave structure, exact dyadic
  values, strict ascent.
* the comparison: on N(0, 0.02) weights, the oracle's round trip
  (quantize, double quant, dequant) has a smaller RMS error with NF4 than
  with INT4 or FP4, for each constant map.
"""
import numpy as np
import pytest

import oracle
from oracle import codebooks as cb
from bit_quantized_lora_blockwise_b200.inputs import bf16_bits, weight_bf16


def test_int4_midpoint_rule_is_absmax_rounding():
    lv = cb.int4_levels()
    x = np.linspace(-1.0, 1.0, 20001, dtype=np.float64).astype(np.float32)
    mids = ((lv[:-1].astype(np.float32) + lv[1:]) * np.float32(0.5)).astype(np.float32)
    t = 7.0 * x.astype(np.float64)
    not_tie = np.abs(t - np.floor(t) - 0.5) > 1e-4
    for xi in x[not_tie][::97]:
        code = oracle.nearest_level(float(xi), lv)
        assert code == int(np.floor(7.0 * float(xi) + 0.5)) + 8
        assert code == int(np.count_nonzero(mids < xi))
    assert np.all(np.diff(lv) > 0) and lv[8] == 0.0 and lv[15] == 1.0


def _e2m1(bits: int) -> float:
    s, e, m = (bits >> 3) & 1, (bits >> 1) & 3, bits & 1
    mag = (m * 0.5) if e == 0 else (1.0 + 0.5 * m) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_fp4_levels_are_e2m1_over_its_maximum():
    vals = sorted({_e2m1(b) for b in range(16)})  # -0 and +0 compare equal: 15 values
    assert len(vals) == 15 and max(vals) == 6.0
    lv = cb.fp4_levels()
    assert np.array_equal(lv[:15], np.array([v / 6.0 for v in vals], np.float32))
    assert lv[15] > 1.0 and (lv[14] + lv[15]) / 2 > 1.0  # the padding level is never the nearest
    assert np.signbit(lv[7]) == False and lv[7] == 0.0
    assert np.all(np.diff(lv) > 0)


def test_dq_signed_map():
    t = cb.dq_signed_levels()
    assert t[0] == -1.0 and t[255] == 1.0 and np.all(np.diff(t) > 0)
    assert np.array_equal(t, -t[::-1])
    assert np.allclose(np.diff(t.astype(np.float64)), 2.0 / 255.0, rtol=0, atol=1e-7)


def test_dq_dynamic_map():
    t = cb.dq_dynamic_levels()
    assert t[0] == 0.0 and t[255] == 1.0 and np.all(np.diff(t) > 0)
    for v in t.astype(np.float64):
        num, den = float(v).as_integer_ratio()
        assert den & (den - 1) == 0, "every level is a dyadic rational"
    top = t[-32:].astype(np.float64)  # the top octave: 33/64 .. 1 in steps of 1/64
    assert np.allclose(np.diff(top), 1.0 / 64.0, rtol=0, atol=0)


@pytest.fixture(scope="module")
def roundtrip_rmse():
    W = weight_bf16(64, 16384, 0.02, 7)
    bits = bf16_bits(W)
    w = oracle.bf16_to_f32(bits).astype(np.float64).reshape(-1)
    out = {}
    for name, lv in (("nf4", oracle.nf4_levels()), ("int4", cb.int4_levels()), ("fp4", cb.fp4_levels())):
        for tname, t8 in (("linear", oracle.dq_levels()), ("signed", cb.dq_signed_levels()),
                          ("dynamic", cb.dq_dynamic_levels())):
            pk, am = oracle.quantize_nf4(bits, lv)
            q, s2 = oracle.double_quant(am, t8)
            wq = oracle.bf16_to_f32(oracle.dequant(pk, q, s2, w.size, lv, t8)).astype(np.float64)
            out[(name, tname)] = float(np.sqrt(np.mean((wq - w) ** 2)))
    return out


@pytest.mark.parametrize("t8", ["linear", "signed", "dynamic"])
def test_nf4_has_the_smallest_roundtrip_error(roundtrip_rmse, t8):
    e = {k: v for (k, t), v in roundtrip_rmse.items() if t == t8}
    print(t8, {k: round(v / 0.02, 5) for k, v in e.items()})
    assert e["nf4"] < e["fp4"] and e["nf4"] < e["int4"]


def test_linear_constant_map_is_the_most_accurate(roundtrip_rmse):
    for name in ("nf4", "int4", "fp4"):
        assert roundtrip_rmse[(name, "linear")] <= roundtrip_rmse[(name, "signed")]
        assert roundtrip_rmse[(name, "linear")] <= roundtrip_rmse[(name, "dynamic")]
