"""Pins of the straight-through backward oracle (oracle/backward.py): brute
force with exactly rounded sums, the matmul rule's special cases, and the
page's choice of the float32 masters over the dequantized weights."""
import math

import numpy as np
import pytest

import oracle
from oracle import backward
from workloads import random_problem

F32 = np.float32


@pytest.mark.parametrize("M,N,K", [(3, 4, 5), (1, 7, 2), (6, 1, 9), (4, 4, 4)])
def test_brute_force_fsum(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    dY = rng.standard_normal((M, N)).astype(F32)
    X = rng.standard_normal((M, K)).astype(F32)
    W = (rng.standard_normal((N, K)) * 0.02).astype(F32)
    dX, dW, db = backward.ste_backward(dY, X, W)
    for m in range(M):
        for k in range(K):
            ref = math.fsum(float(dY[m, n]) * float(W[n, k]) for n in range(N))
            assert abs(dX[m, k] - ref) <= 1e-15 * max(1.0, abs(ref))
    for n in range(N):
        for k in range(K):
            ref = math.fsum(float(dY[m, n]) * float(X[m, k]) for m in range(M))
            assert abs(dW[n, k] - ref) <= 1e-15 * max(1.0, abs(ref))
        assert abs(db[n] - math.fsum(float(dY[m, n]) for m in range(M))) <= 1e-15


def test_special_cases():
    """Identity weights pass dL/dy straight through; a one-hot input row copies
    dL/dy into one column of dL/dW; all-ones dL/dy sums W's columns."""
    rng = np.random.default_rng(1)
    dY = rng.standard_normal((3, 5)).astype(F32)
    dX, _, db = backward.ste_backward(dY, rng.standard_normal((3, 5)).astype(F32), np.eye(5, dtype=F32))
    np.testing.assert_array_equal(dX, dY.astype(np.float64))
    np.testing.assert_allclose(db, dY.astype(np.float64).sum(0), rtol=0, atol=1e-15)
    X = np.zeros((3, 4), F32)
    X[:, 2] = 1.0
    _, dW, _ = backward.ste_backward(dY, X, rng.standard_normal((5, 4)).astype(F32))
    np.testing.assert_allclose(dW[:, 2], dY.astype(np.float64).sum(0), rtol=0, atol=1e-15)
    assert np.all(dW[:, [0, 1, 3]] == 0)
    W = rng.standard_normal((5, 4)).astype(F32)
    dX1, _, db1 = backward.ste_backward(np.ones((2, 5), F32), np.zeros((2, 4), F32), W)
    np.testing.assert_allclose(dX1[0], W.astype(np.float64).sum(0), rtol=1e-15)
    assert db1.tolist() == [2.0] * 5


def test_uses_the_float32_masters_not_the_dequantized_weights():
    """Straight through: dL/dx flows through W itself, so it differs from the
    product with beta W_q (the quantizer treated as the identity)."""
    p = random_problem(5, 4, 64, 32)
    dY = np.random.default_rng(2).standard_normal((4, 32)).astype(F32)
    dX, _, _ = backward.ste_backward(dY, p.X, p.W)
    beta = oracle.absmean_beta(p.W, 1e-5)
    deq = oracle.ternarize(p.W, beta).astype(np.float64) * float(beta)
    assert not np.allclose(dX, dY.astype(np.float64) @ deq, rtol=1e-3)
    np.testing.assert_allclose(dX, dY.astype(np.float64) @ p.W.astype(np.float64), rtol=1e-12)


def test_abs_bound_dominates():
    rng = np.random.default_rng(3)
    dY, X, W = (rng.standard_normal(s).astype(F32) for s in ((5, 6), (5, 7), (6, 7)))
    outs, bounds = backward.ste_backward(dY, X, W), backward.abs_bound(dY, X, W)
    for o, b in zip(outs, bounds):
        assert np.all(np.abs(o) <= b + 1e-12)
    assert backward.abs_bound(np.ones((2, 3), F32), np.ones((2, 4), F32), -np.ones((3, 4), F32))[0].tolist() == \
        [[3.0] * 4] * 2


def test_rejects_mismatched_shapes():
    with pytest.raises(ValueError):
        backward.ste_backward(np.zeros((2, 3), F32), np.zeros((2, 4), F32), np.zeros((4, 4), F32))
