"""Pins of the oracle's linear layer (float64).

* forward Y = X W'^T + s (X A) B against naive Python loops on tiny shapes
  (brute force);
* backward dX, dA, dB against central finite differences of the scalar
  L = <dY, Y> (the layer is linear in X, A and B, so the differences are
  exact up to rounding);
* B = 0 reproduces the quantized base exactly and gives dA = 0; A = 0 gives
  dB = 0 (intvml.com "DL0087 QLoRA", formulation list: with the adapter B
  at its zero initial value the layer equals the quantized base);
* a planted mistake (an operand transposed in a copy of the backward) is
  caught by the finite-difference pin.
"""
import itertools

import numpy as np
import pytest

import oracle


def _naive_fwd(X, W, A, B, s):
    M, K = len(X), len(X[0])
    N, r = len(W), len(A[0])
    Y = [[0.0] * N for _ in range(M)]
    for i in range(M):
        xa = [sum(X[i][k] * A[k][t] for k in range(K)) for t in range(r)]
        for j in range(N):
            Y[i][j] = sum(X[i][k] * W[j][k] for k in range(K)) + s * sum(xa[t] * B[t][j] for t in range(r))
    return np.array(Y)


@pytest.mark.parametrize("M,N,K,r", [(m, n, k, r) for m, n, k, r in
                                     itertools.product([1, 2, 3], [64, 128], [64, 128], [1, 8])
                                     if (m, n, k) in ((1, 64, 64), (2, 128, 64), (3, 64, 128), (3, 128, 128))])
def test_fwd_against_naive_loops(M, N, K, r):
    rng = np.random.default_rng(M * 1000 + N + K + r)
    X, W = rng.standard_normal((M, K)), rng.standard_normal((N, K))
    A, B = rng.standard_normal((K, r)), rng.standard_normal((r, N))
    alpha = 16.0
    Y, XA = oracle.linear_fwd(X, W, A, B, alpha, r)
    ref = _naive_fwd(X.tolist(), W.tolist(), A.tolist(), B.tolist(), alpha / r)
    assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12)
    assert np.allclose(XA, X @ A, rtol=1e-12, atol=1e-12)


def _fd_check(bwd, M=3, N=5, K=4, r=2, alpha=6.0):
    rng = np.random.default_rng(11)
    X, W = rng.standard_normal((M, K)), rng.standard_normal((N, K))
    A, B = rng.standard_normal((K, r)), rng.standard_normal((r, N))
    dY = rng.standard_normal((M, N))

    def loss(X_, A_, B_):
        return float(np.sum(dY * oracle.linear_fwd(X_, W, A_, B_, alpha, r)[0]))

    dX, dA, dB = bwd(X, dY, W, A, B, alpha, r)
    h = 1e-5
    ok = True
    for name, arr, grad in (("X", X, dX), ("A", A, dA), ("B", B, dB)):
        fd = np.zeros_like(arr)
        for idx in np.ndindex(arr.shape):
            p, m = arr.copy(), arr.copy()
            p[idx] += h
            m[idx] -= h
            args_p = {"X": (p, A, B), "A": (X, p, B), "B": (X, A, p)}[name]
            args_m = {"X": (m, A, B), "A": (X, m, B), "B": (X, A, m)}[name]
            fd[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        ok &= bool(np.allclose(fd, grad, rtol=1e-7, atol=1e-8))
    return ok


def test_bwd_finite_differences():
    assert _fd_check(oracle.linear_bwd)


def test_planted_mistake_is_caught():
    def broken(X, dY, W, A, B, alpha, r):
        dX, dA, dB = oracle.linear_bwd(X, dY, W, A, B, alpha, r)
        s = alpha / r
        G = dY @ B.T
        return dX, s * (X.T @ G), np.flip(dB, axis=1)  # dB columns reversed
    assert not _fd_check(broken)

    def dropped_scale(X, dY, W, A, B, alpha, r):
        dX, dA, dB = oracle.linear_bwd(X, dY, W, A, B, alpha, r)
        return dX, dA * (r / alpha), dB
    assert not _fd_check(dropped_scale)


def test_B_zero_reproduces_base_and_zero_grads():
    rng = np.random.default_rng(3)
    M, N, K, r = 4, 64, 128, 8
    X, W = rng.standard_normal((M, K)), rng.standard_normal((N, K))
    A, B = rng.standard_normal((K, r)), np.zeros((r, N))
    dY = rng.standard_normal((M, N))
    Y, _ = oracle.linear_fwd(X, W, A, B, 16.0, r)
    assert np.array_equal(Y, X @ W.T)
    dX, dA, dB = oracle.linear_bwd(X, dY, W, A, B, 16.0, r)
    assert np.all(dA == 0.0)
    assert np.array_equal(dX, dY @ W)
    dX, dA, dB = oracle.linear_bwd(X, dY, W, np.zeros((K, r)), rng.standard_normal((r, N)), 16.0, r)
    assert np.all(dB == 0.0)


def test_rows_variants_agree_with_full():
    rng = np.random.default_rng(9)
    M, N, K, r = 6, 64, 128, 8
    X, W = rng.standard_normal((M, K)), rng.standard_normal((N, K))
    A, B = rng.standard_normal((K, r)), rng.standard_normal((r, N))
    dY = rng.standard_normal((M, N))
    rows = np.array([0, 3, 5])
    Y, _ = oracle.linear_fwd(X, W, A, B, 16.0, r)
    assert np.allclose(oracle.linear_fwd_rows(rows, X, W, A, B, 16.0, r), Y[rows], rtol=1e-13)
    dX, dA, dB = oracle.linear_bwd(X, dY, W, A, B, 16.0, r)
    dXr, dA2, dB2 = oracle.linear_bwd_rows(rows, X, dY, W, A, B, 16.0, r)
    assert np.allclose(dXr, dX[rows], rtol=1e-13)
    assert np.allclose(dA2, dA) and np.allclose(dB2, dB)
