"""Pins for the CPU oracle: it is checked against things other than itself.

Hand-worked dyadic cases (tests/golden/hand_worked.json), closed forms,
invariants, exact-rational brute force and special cases.  Each test names the
kind of mistake it is there to catch.
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from workloads import random_problem

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "hand_worked.json")) as fh:
    GOLD = json.load(fh)
F32 = np.float32


# ---------------------------------------------------------------- weights ---
@pytest.mark.parametrize("case", GOLD["weights"], ids=lambda c: c["name"])
def test_weights_hand_worked(case):
    W = np.array(case["W"], F32)
    beta = oracle.absmean_beta(W, case["eps"])
    assert float(beta) == case["beta"]
    np.testing.assert_array_equal(oracle.ternarize(W, beta), np.array(case["Wq"], np.int8))


def _fraction_beta(W, eps):
    """beta by exact rational arithmetic (a different algorithm from math.fsum)."""
    S = sum((Fraction(float(v)) for v in np.abs(W.astype(F32)).ravel()), Fraction(0))
    D = float(S)                      # int/Fraction -> float is correctly rounded
    return F32(F32(D / W.size) + F32(eps))


@pytest.mark.parametrize("seed", range(6))
def test_beta_is_exact_mean(seed):
    """Catches a float32 running sum, a dropped element or a wrong n."""
    rng = np.random.default_rng(100 + seed)
    n, k = int(rng.integers(1, 40)), int(rng.integers(1, 70))
    W = (rng.standard_normal((n, k)) * 10.0 ** rng.integers(-6, 3)).astype(F32)
    if seed % 2:  # wide dynamic range: naive summation loses the small terms
        W.ravel()[:: 3] *= F32(2.0 ** 40)
        W.ravel()[1:: 5] *= F32(2.0 ** -60)
    assert oracle.absmean_beta(W, 1e-5) == _fraction_beta(W, 1e-5)


def test_beta_closed_form_constant_tensor():
    """mean of n equal values is the value: a float32 running sum drifts here."""
    c = F32(0.02)
    W = np.full((1001, 999), c, F32)
    assert oracle.absmean_beta(W, 1e-5) == F32(c + F32(1e-5))
    assert np.all(oracle.ternarize(W, oracle.absmean_beta(W, 1e-5)) == 1)
    assert np.all(oracle.ternarize(-W, oracle.absmean_beta(-W, 1e-5)) == -1)


def test_beta_is_per_tensor_and_sign_blind():
    rng = np.random.default_rng(7)
    W = rng.standard_normal((16, 33)).astype(F32)
    b = oracle.absmean_beta(W, 1e-5)
    assert oracle.absmean_beta(-W, 1e-5) == b
    assert oracle.absmean_beta(W[::-1, ::-1].copy(), 1e-5) == b   # order-free
    assert oracle.absmean_beta(W.T.copy(), 1e-5) == b


def test_ternary_codes_and_zero_fraction_gaussian():
    """Closed form: for Gaussian W, P(|Z| < E|Z|/2) = erf(sqrt(2/pi)/2/sqrt(2)) = 0.3101.

    The 31% zero trits quoted on "a 1-bit llm, from scratch" (tl;dr)."""
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((1000, 1000)) * 0.02).astype(F32)
    Wq = oracle.ternarize(W, oracle.absmean_beta(W, 1e-5))
    assert set(np.unique(Wq)) <= {-1, 0, 1}
    p0 = math.erf(0.5 * math.sqrt(2 / math.pi) / math.sqrt(2))
    assert abs(np.mean(Wq == 0) - p0) < 0.003
    assert abs(np.mean(Wq == 1) - np.mean(Wq == -1)) < 0.004
    # a sign error in the code would flip this correlation
    assert np.all(np.sign(W[Wq != 0]) == Wq[Wq != 0])


def test_ternary_fractions_uniform():
    """U(-a,a): E|w| = a/2, so zeros are |w| < a/4: 25% zeros, 37.5% each sign."""
    rng = np.random.default_rng(12)
    W = ((rng.random((1000, 1000), dtype=F32) * 2 - 1) * F32(0.05)).astype(F32)
    Wq = oracle.ternarize(W, oracle.absmean_beta(W, 1e-5))
    assert abs(np.mean(Wq == 0) - 0.25) < 0.003
    assert abs(np.mean(Wq == 1) - 0.375) < 0.003


def test_ternarize_scale_invariance():
    """W*4 with eps -> 0 gives the same codes (beta scales with W)."""
    rng = np.random.default_rng(13)
    W = rng.standard_normal((64, 64)).astype(F32)
    a = oracle.ternarize(W, oracle.absmean_beta(W, 2.0 ** -60))
    b = oracle.ternarize(W * F32(4), oracle.absmean_beta(W * F32(4), 2.0 ** -58))
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------------------ activations ---
@pytest.mark.parametrize("case", GOLD["activations"], ids=lambda c: c["name"])
def test_act_quant_hand_worked(case):
    X = np.array(case["X"], F32)
    Xq, s = oracle.act_quant(X, case["eps"])
    np.testing.assert_array_equal(Xq, np.array(case["Xq"], np.int8))
    if "s_exact" in case:
        assert float(s[0]) == case["s_exact"]
    else:
        assert abs(float(s[0]) - case["s_real"]) <= case["s_rel_tol"] * case["s_real"]


def test_act_quant_invariants():
    rng = np.random.default_rng(21)
    X = (rng.standard_normal((50, 300)) * rng.uniform(0.3, 50, (50, 1))).astype(F32)
    Xq, s = oracle.act_quant(X, 1e-5)
    assert Xq.dtype == np.int8 and Xq.min() >= -127 and Xq.max() <= 127
    # the row maximum lands on code 126 or 127 (s is slightly above max/127)
    i = np.argmax(np.abs(X), axis=1)
    top = np.abs(Xq[np.arange(50), i].astype(int))
    assert np.all((top == 127) | (top == 126))
    # scale is per row: equals max/127 to within float32 rounding plus eps
    ref = np.max(np.abs(X.astype(np.float64)), axis=1) / 127 + 1e-5
    assert np.allclose(s, ref, rtol=3e-7, atol=0)
    # dequantized codes approximate X to within half a step per element
    assert np.all(np.abs(Xq * s[:, None].astype(np.float64) - X) <= s[:, None] * 0.5 + 1e-6)


def test_act_quant_row_independence():
    """Per-row scales: perturbing row j leaves every other row bit-identical
    ("attention, as graph ops": a per-tensor max lets the future leak)."""
    rng = np.random.default_rng(22)
    X = rng.standard_normal((9, 40)).astype(F32)
    Xq, s = oracle.act_quant(X, 1e-5)
    Y = X.copy()
    Y[4] *= F32(1000)
    Y[4, 3] = F32(-7e5)
    Yq, t = oracle.act_quant(Y, 1e-5)
    keep = [r for r in range(9) if r != 4]
    np.testing.assert_array_equal(Xq[keep], Yq[keep])
    np.testing.assert_array_equal(s[keep], t[keep])


# ---------------------------------------------------------------- packing ---
@pytest.mark.parametrize("case", GOLD["packing"], ids=lambda c: str(c["trits"]))
def test_pack_hand_worked(case):
    t = np.array([case["trits"]], np.int8)
    p = oracle.pack5(t, ldp=1)
    assert int(p[0, 0]) == case["byte"]
    np.testing.assert_array_equal(oracle.unpack5(p, 5), t)


def test_pack_is_a_bijection_on_all_243_patterns():
    pats = np.array(list(itertools.product((-1, 0, 1), repeat=5)), np.int8)
    bytes_ = oracle.pack5(pats, ldp=1)[:, 0].astype(int)
    assert sorted(bytes_.tolist()) == list(range(243))
    np.testing.assert_array_equal(oracle.unpack5(bytes_.reshape(-1, 1).astype(np.uint8), 5), pats)
    # digit k has weight 3^k: flipping trit k from -1 to 0 adds exactly 3^k
    for k in range(5):
        a = np.full((1, 5), -1, np.int8)
        b = a.copy()
        b[0, k] = 0
        assert int(oracle.pack5(b, 1)[0, 0]) - int(oracle.pack5(a, 1)[0, 0]) == 3 ** k


@pytest.mark.parametrize("K", [1, 4, 5, 6, 7, 79, 80, 81, 128, 2560, 6912])
def test_pack_roundtrip_and_padding(K):
    rng = np.random.default_rng(K)
    t = rng.integers(-1, 2, (3, K)).astype(np.int8)
    ldp = oracle.pack5_ldp(K)
    assert ldp % 16 == 0 and ldp * 5 >= K and (ldp - 16) * 5 < K
    p = oracle.pack5(t, ldp)
    assert p.shape == (3, ldp) and p.max() <= 242
    np.testing.assert_array_equal(oracle.unpack5(p, K), t)
    nb = -(-K // 5)
    assert np.all(p[:, nb:] == 121)          # whole padding bytes: all-zero trits
    if K % 5:                                 # the ragged byte's high digits are 1
        hi = p[:, nb - 1].astype(int) // 3 ** (K % 5)
        assert np.all(hi == (3 ** (5 - K % 5) - 1) // 2)


def test_pack_ldp_values():
    assert [oracle.pack5_ldp(k) for k in (128, 2560, 4096, 6912, 8192, 11008)] == \
        [32, 512, 832, 1392, 1648, 2208]


# ------------------------------------------------------------ contraction ---
@pytest.mark.parametrize("M,N,K", [(3, 4, 11), (3, 6, 6)])
def test_contract_brute_force_loops(M, N, K):
    rng = np.random.default_rng(31 + K)
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    Wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
    acc = oracle.contract(Xq, Wq)
    for m in range(M):
        for n in range(N):
            tot = 0
            for k in range(K):
                w = int(Wq[n, k])
                if w == 1:
                    tot += int(Xq[m, k])        # add
                elif w == -1:
                    tot -= int(Xq[m, k])        # subtract (zero: skip)
            assert acc[m, n] == tot
    idx_m, idx_n = np.array([0, 2, 1]), np.array([3, 0, 2])
    np.testing.assert_array_equal(oracle.contract_entries(Xq[idx_m], Wq[idx_n]), acc[idx_m, idx_n])


def test_contract_extremes():
    K = 8192
    Xq = np.full((2, K), 127, np.int8)
    Xq[1] = -127
    Wq = np.ones((2, K), np.int8)
    Wq[1] = -1
    acc = oracle.contract(Xq, Wq)
    assert acc.tolist() == [[127 * K, -127 * K], [-127 * K, 127 * K]]


def test_contract_f64_equals_integer_contract():
    """The float64 product of the codes is the exact integer product: random
    codes, the extremes, and a column-sliced (transposition-sensitive) case."""
    rng = np.random.default_rng(57)
    for M, N, K in ((7, 5, 33), (16, 16, 1000), (3, 40, 6912)):
        Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        Wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
        np.testing.assert_array_equal(oracle.contract_f64(Xq, Wq), oracle.contract(Xq, Wq))
        np.testing.assert_array_equal(oracle.contract_f64(Xq[:, :K // 2], Wq[:, :K // 2]),
                                      oracle.contract(Xq[:, :K // 2], Wq[:, :K // 2]))
    K = 131072
    Xq = np.full((2, K), 127, np.int8)
    Xq[1] = -127
    Wq = np.ones((2, K), np.int8)
    Wq[1, ::2] = -1
    acc = oracle.contract_f64(Xq, Wq)
    assert acc.tolist() == [[127 * K, 0], [-127 * K, 0]]
    sq = rng.integers(-1, 2, (9, 9)).astype(np.int8)
    xs = rng.integers(-127, 128, (4, 9)).astype(np.int8)
    assert np.array_equal(oracle.contract_f64(xs, sq), oracle.contract(xs, sq))


# ---------------------------------------------------------------- dequant ---
@pytest.mark.parametrize("case", GOLD["dequant"], ids=lambda c: c["name"])
def test_dequant_hand_worked(case):
    acc = np.array(case["acc"], np.int32)
    s = np.array(case["s"], F32)
    y = oracle.dequant(acc, s, F32(case["beta"]))
    np.testing.assert_array_equal(y, np.array(case["Y_nobias"], F32))
    if case.get("bias") is not None:
        yb = oracle.dequant(acc, s, F32(case["beta"]), np.array(case["bias"], F32))
        np.testing.assert_array_equal(yb, np.array(case["Y_bias"], F32))


# ------------------------------------------------------------- whole layer --
@pytest.mark.parametrize("shape", [(1, 7, 3), (4, 16, 5), (2, 13, 16), (5, 1, 2)])
def test_layer_brute_force_fp64(shape):
    """y = sum_k (s x_q)(beta w_q) in float64 matches the float32 layer to 1e-6."""
    M, K, N = shape
    p = random_problem(40 + K, M, K, N, w_sigma=0.5)
    r = oracle.bitlinear(p.X, p.W, 1e-5)
    xd = r["Xq"].astype(np.float64) * r["s"].astype(np.float64)[:, None]
    wd = r["Wq"].astype(np.float64) * float(r["beta"])
    ybf = xd @ wd.T
    err = np.abs(r["Y"] - ybf)
    assert np.all(err <= 1e-6 * np.maximum(np.abs(ybf), 1e-30) + 1e-30)


def test_layer_one_hot_row():
    """X = c e_k: x_q = 127 e_k and y = 127 W_q[:, k] (s beta)."""
    rng = np.random.default_rng(51)
    W = (rng.standard_normal((6, 9)) * 0.02).astype(F32)
    X = np.zeros((1, 9), F32)
    X[0, 4] = 3.0
    r = oracle.bitlinear(X, W, 1e-5)
    assert r["Xq"].tolist() == [[0, 0, 0, 0, 127, 0, 0, 0, 0]]
    np.testing.assert_array_equal(r["acc"][0], 127 * r["Wq"][:, 4].astype(np.int32))
    sb = F32(r["s"][0] * r["beta"])
    np.testing.assert_array_equal(r["Y"][0], (127 * r["Wq"][:, 4]).astype(F32) * sb)


def test_layer_batched_equals_row_by_row():
    """A cached decode step equals the full forward at that position
    (ultragraph-1bit, 'A mesh of minds': per-token quantization)."""
    p = random_problem(52, 6, 40, 7)
    full = oracle.bitlinear(p.X, p.W, 1e-5)["Y"]
    for m in range(6):
        one = oracle.bitlinear(p.X[m:m + 1], p.W, 1e-5)["Y"]
        np.testing.assert_array_equal(one[0], full[m])


def test_rejects_nonfinite():
    W = np.ones((2, 2), F32)
    W[0, 0] = np.inf
    with pytest.raises(ValueError):
        oracle.absmean_beta(W, 1e-5)
    with pytest.raises(ValueError):
        oracle.act_quant(np.array([[np.nan, 1.0]], F32), 1e-5)
