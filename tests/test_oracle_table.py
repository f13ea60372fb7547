"""Pins of the oracle's code tables against what the pages fix.

NF4 (promptingindex.com "4-bit NormalFloat"; intvml.com "DL0087 QLoRA",
formulation symbol list): 16 levels, at quantiles of the standard normal,
equal probability mass per level, rescaled to [-1, 1], with an exact zero.
The construction is cross-checked against Python's own normal quantile
(statistics.NormalDist.inv_cdf, Wichura's AS241), a routine independent of
the oracle's bisection on erfc. The exact level values are not printed on
the pages: agreement with any external NF4 table is not claimed.
"""
import json
import os
from statistics import NormalDist

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore")

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_figures.json")))
DELTA = 0.5 * ((1 - 1 / 30) + (1 - 1 / 32))


def test_nf4_table_fixed_properties():
    L = oracle.nf4_levels()
    g = GOLDEN["nf4_levels"]
    assert L.dtype == np.float32 and L.shape == (g["count"],)
    assert np.all(np.diff(L) > 0), "levels must be strictly ascending"
    assert L[0] == np.float32(g["min"]) and L[-1] == np.float32(g["max"])
    assert L[7] == 0.0 and np.signbit(L[7]) == False  # exact +0
    assert int((L < 0).sum()) == 7 and int((L > 0).sum()) == 8


def test_nf4_equal_probability_mass_each_side():
    """Phi(L_i * z(delta)) is evenly spaced on each side of zero: each level
    covers the same probability mass (promptingindex.com, NF4 section)."""
    nd = NormalDist()
    L = oracle.nf4_levels().astype(np.float64)
    z = nd.inv_cdf(DELTA)
    pos = np.array([nd.cdf(v * z) for v in L[8:]])         # ascending
    neg = np.array([nd.cdf(-v * z) for v in L[:7]])        # descending
    assert np.allclose(np.diff(pos), (DELTA - 0.5) / 8, atol=2e-7)
    assert np.allclose(np.diff(neg), -(DELTA - 0.5) / 7, atol=2e-7)
    assert abs(pos[-1] - DELTA) < 1e-7 and abs(neg[0] - DELTA) < 1e-7


def test_nf4_matches_independent_quantile_routine():
    nd = NormalDist()
    z = nd.inv_cdf(DELTA)
    ref = [-nd.inv_cdf(DELTA + i * (0.5 - DELTA) / 7) / z for i in range(7)] + [0.0] + \
          [nd.inv_cdf(DELTA + j * (0.5 - DELTA) / 8) / z for j in range(7, -1, -1)]
    ref = np.array(ref, dtype=np.float64)
    L = oracle.nf4_levels().astype(np.float64)
    # within one fp32 ulp of the independently computed value
    ulp = np.spacing(np.abs(ref).astype(np.float32)).astype(np.float64)
    assert np.all(np.abs(L - ref) <= ulp)


def test_dq_table_linear_unsigned():
    T = oracle.dq_levels()
    assert T.shape == (256,) and T.dtype == np.float32
    assert T[0] == 0.0 and T[255] == 1.0
    assert np.all(np.diff(T) > 0)
    expect = (np.arange(256, dtype=np.float64) / 255.0).astype(np.float32)
    assert np.array_equal(T, expect)
