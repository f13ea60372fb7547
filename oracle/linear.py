"""float64 oracle for the QLoRA linear layer (test infrastructure only).

The layer, as the pages describe it (intvml.com "DL0087 QLoRA: 4-bit
Quantized LoRA", opening paragraph, Figure 1 and the formulation's symbol
list; sandgarden.com "QLoRA", workflow step "Fine-Tune the Adapters"):

* forward: the frozen NF4 weight is dequantized to bf16 (W'), used for the
  matmul, and the low-rank update of the bf16 adapters A [K, r] and
  B [r, N], scaled by s = alpha / r, is added:
      Y = X W'^T + s (X A) B
* backward: gradients pass through the frozen W' into the adapters only
  (no gradient for W):
      G  = dY B^T
      dX = dY W' + s G A^T
      dA = s X^T G
      dB = s (X A)^T dY

All inputs are bf16 bit patterns (uint16) and are widened exactly to
float64; every product and sum is float64 (numpy matmul is the library
primitive used for each product, in the order written above).
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _f64(a):
    a = np.asarray(a)
    return bf16_bits_to_f64(a) if a.dtype == np.uint16 else a.astype(np.float64)


def linear_fwd(X, W, A, B, alpha: float, r: int):
    """Y [M,N] and XA [M,r] in float64. W is the dequantized weight [N,K]."""
    X, W, A, B = map(_f64, (X, W, A, B))
    s = float(alpha) / float(r)
    XA = X @ A
    Y = X @ W.T + s * (XA @ B)
    return Y, XA


def linear_fwd_rows(rows, X, W, A, B, alpha: float, r: int):
    """Rows `rows` of Y only (same arithmetic as linear_fwd)."""
    rows = np.asarray(rows)
    X = _f64(np.asarray(X)[rows])
    W, A, B = map(_f64, (W, A, B))
    s = float(alpha) / float(r)
    return X @ W.T + s * ((X @ A) @ B)


def linear_bwd(X, dY, W, A, B, alpha: float, r: int):
    """dX [M,K], dA [K,r], dB [r,N] in float64 (no dW: W is frozen)."""
    X, dY, W, A, B = map(_f64, (X, dY, W, A, B))
    s = float(alpha) / float(r)
    G = dY @ B.T
    dX = dY @ W + s * (G @ A.T)
    dA = s * (X.T @ G)
    dB = s * ((X @ A).T @ dY)
    return dX, dA, dB


def linear_bwd_rows(rows, X, dY, W, A, B, alpha: float, r: int):
    """dA and dB in full (they reduce over every token) and rows `rows` of dX."""
    rows = np.asarray(rows)
    X, dY, W, A, B = map(_f64, (X, dY, W, A, B))
    s = float(alpha) / float(r)
    G = dY @ B.T
    dXr = dY[rows] @ W + s * (G[rows] @ A.T)
    dA = s * (X.T @ G)
    dB = s * ((X @ A).T @ dY)
    return dXr, dA, dB
