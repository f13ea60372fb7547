"""float64 oracle of one AdamW step (test infrastructure only).

The pages name paged optimizers for the adapters (intvml.com "DL0087 QLoRA:
4-bit Quantized LoRA", component (5); promptingindex.com "QLoRA: Finetuning
65B Models on a Single GPU", "Double Quantization and Paged Optimizers")
without restating the optimizer; the optimizer is AdamW with decoupled
weight decay as published (I. Loshchilov and F. Hutter, "Decoupled Weight
Decay Regularization", ICLR 2019, Algorithm 2, with the schedule multiplier
folded into the learning rate), written here step by step:

    p <- p (1 - lr wd)                      decoupled decay
    m <- b1 m + (1 - b1) g                  first moment
    v <- b2 v + (1 - b2) g^2                second moment
    m_hat = m / (1 - b1^t),  v_hat = v / (1 - b2^t)
    p <- p - lr m_hat / (sqrt(v_hat) + eps)
"""
from __future__ import annotations

import numpy as np


def adamw_step(p, m, v, g, t: int, lr: float, b1: float, b2: float, eps: float, wd: float):
    """One step on float64 arrays; returns the new (p, m, v)."""
    p, m, v, g = (np.asarray(a, np.float64) for a in (p, m, v, g))
    p = p * (1.0 - lr * wd)
    m = b1 * m + (1.0 - b1) * g
    v = b2 * v + (1.0 - b2) * g * g
    m_hat = m / (1.0 - b1 ** t)
    v_hat = v / (1.0 - b2 ** t)
    p = p - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p, m, v
