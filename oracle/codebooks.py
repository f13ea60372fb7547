"""Alternative code tables for the QLoRA codec (test infrastructure only).

The QLoRA pages compare the 4-bit NormalFloat type with the uniform 4-bit
types it outperforms (promptingindex.com "Finetuning 65B Models on a Single
GPU", section "4-bit NormalFloat": NF4 beats 4-bit integers and 4-bit
floats; intvml.com "DL0087 QLoRA", component (1)). The codec takes its level
tables as inputs, so these types are table swaps. Each table here is built
from its own definition, in float64, then rounded once to float32:

* int4_levels   symmetric absmax 4-bit integers: code i in -8..7 stands for
                i / 7 (x in [-1, 1] rounds to one of the 15 levels i / 7 with
                |i| <= 7; -8/7 lies below -1 and is never the nearest level).
* fp4_levels    the E2M1 4-bit float (1 sign, 2 exponent bits with bias 1,
                1 mantissa bit; values 0, 0.5, 1, 1.5, 2, 3, 4, 6 and their
                negatives) divided by its largest value 6, so the range is
                [-1, 1]; +0 and -0 are one level, and a sixteenth level 8/6,
                above 1 and never the nearest, keeps the table at 16 ascending
                entries.
* dq_signed_levels   an 8-bit signed linear map (2k - 255) / 255, k = 0..255,
                     over [-1, 1]: the block constants are non-negative, so
                     only its upper half is ever used.
* dq_dynamic_levels  an 8-bit dynamic-exponent map over [0, 1]: 0, then for
                     j = 0..254 the values 2^-e (1 - m/64) with
                     (e, m) = divmod(j, 32): 8 octaves of 32 linearly spaced
                     levels each, every one an exact dyadic rational.

The mean-centred 8-bit map would store a per-group mean besides the scale;
the storage count on the pages (4 + 8/64 + 32/(64*256) bits per parameter)
has no room for it, so it is not built.
"""
from __future__ import annotations

import numpy as np


def int4_levels() -> np.ndarray:
    return np.array([i / 7.0 for i in range(-8, 8)], dtype=np.float32)


def fp4_levels() -> np.ndarray:
    mags = [0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    vals = [-m for m in reversed(mags)] + [0.0] + mags  # 15 values: -0 and +0 are one level, +0
    vals.append(8.0)  # padding level above the range
    return np.array([v / 6.0 for v in vals], dtype=np.float32)


def dq_signed_levels() -> np.ndarray:
    return np.array([(2 * k - 255) / 255.0 for k in range(256)], dtype=np.float32)


def dq_dynamic_levels() -> np.ndarray:
    vals = [0.0]
    for j in range(255):
        e, m = divmod(j, 32)
        vals.append(2.0 ** -e * (1.0 - m / 64.0))
    return np.array(sorted(vals), dtype=np.float32)
