"""Pins of the RMSNorm oracle ("ultragraph -- when the graph is the 1-bit LLM,
part 2", section "attention, as graph ops": RMSNorm(x) = x / sqrt(mean(x^2) +
eps) * g) and of its composition with the per-row activation quantizer."""
import math

import numpy as np
import pytest

import oracle

F32 = np.float32


def test_hand_worked_rows():
    """x = (2,2,2,2): mean of squares 4, 4 + 2^-22 is a float32 tie that rounds
    to the even 4, sqrt 2, so y = g exactly.  x = (3,4,0,0): mean 6.25 (again
    a tie back to 6.25), sqrt 2.5, y = (1.2, 1.6, 0, 0) * g in float32."""
    g = np.array([1, -1, 0.5, 0.25], F32)
    y = oracle.rmsnorm(np.array([[2, 2, 2, 2], [3, 4, 0, 0]], F32), g, 2.0 ** -22)
    np.testing.assert_array_equal(y[0], g)
    np.testing.assert_array_equal(y[1], np.array([F32(1.2), F32(-1.6), 0, 0], F32))


def test_mean_of_squares_is_the_exact_sum():
    """1 followed by 4096 copies of 2^-12: the squares add to exactly 1 + 2^-12,
    which a float32 running sum loses entirely (every 2^-24 is a tie that rounds
    back to 1)."""
    d = 4097
    x = np.full((1, d), F32(2.0 ** -12))
    x[0, 0] = 1.0
    eps = 1e-6
    y = oracle.rmsnorm(x, np.ones(d, F32), eps)
    ms = F32((1.0 + 2.0 ** -12) / d)                   # the exact sum is a float64
    r = np.sqrt(F32(ms + F32(eps)))
    assert y[0, 0] == F32(F32(1.0) / r)
    ms_f32 = F32(F32(1.0) / F32(d))                    # what the running float32 sum would give
    assert y[0, 0] != F32(F32(1.0) / np.sqrt(F32(ms_f32 + F32(eps))))


def test_power_of_two_scaling_is_exact():
    """rmsnorm(2x, g, 4 eps) == rmsnorm(x, g, eps): every step scales exactly."""
    rng = np.random.default_rng(1)
    X = rng.standard_normal((5, 333)).astype(F32)
    g = rng.standard_normal(333).astype(F32)
    np.testing.assert_array_equal(oracle.rmsnorm(2 * X, g, 4e-5), oracle.rmsnorm(X, g, 1e-5))


def test_against_float64_and_unit_rms():
    rng = np.random.default_rng(2)
    X = (rng.standard_normal((7, 1000)) * rng.uniform(0.01, 100, (7, 1))).astype(F32)
    g = rng.uniform(0.5, 2, 1000).astype(F32)
    y = oracle.rmsnorm(X, g, 1e-5)
    x64 = X.astype(np.float64)
    ref = x64 / np.sqrt(np.mean(x64 * x64, axis=1, keepdims=True) + 1e-5) * g.astype(np.float64)
    assert np.max(np.abs(y - ref) / np.abs(ref).max(axis=1, keepdims=True)) < 2.0 ** -21
    y1 = oracle.rmsnorm(X, np.ones(1000, F32), 1e-12).astype(np.float64)
    np.testing.assert_allclose(np.mean(y1 * y1, axis=1), 1.0, rtol=1e-5)


def test_rows_are_independent():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((4, 64)).astype(F32)
    g = rng.standard_normal(64).astype(F32)
    y = oracle.rmsnorm(X, g, 1e-5)
    X2 = X.copy()
    X2[2] *= F32(1e3)
    y2 = oracle.rmsnorm(X2, g, 1e-5)
    np.testing.assert_array_equal(y2[[0, 1, 3]], y[[0, 1, 3]])


def test_norm_then_quantize_hand_worked():
    """y = g = (1, -1, 0.5, 0.25): s = 1/127 + 1e-5; the codes round(y / s) are
    127, -127, 63 (63.42) and 32 (31.71)."""
    g = np.array([1, -1, 0.5, 0.25], F32)
    Xq, s = oracle.rmsnorm_act_quant(np.array([[2, 2, 2, 2]], F32), g, 2.0 ** -22, 1e-5)
    assert s[0] == F32(F32(F32(1.0) / F32(127)) + F32(1e-5))
    assert Xq.tolist() == [[127, -127, 63, 32]]
    for v, c in zip(g, Xq[0]):
        q = float(v) / float(s[0])
        assert abs(q - c) < 0.5 and abs(abs(q - math.floor(q)) - 0.5) > 1e-3


def test_rejects_bad_shapes_and_values():
    with pytest.raises(ValueError):
        oracle.rmsnorm(np.ones((2, 3), F32), np.ones(4, F32), 1e-5)
    with pytest.raises(ValueError):
        oracle.rmsnorm(np.array([[np.inf, 1]], F32), np.ones(2, F32), 1e-5)
