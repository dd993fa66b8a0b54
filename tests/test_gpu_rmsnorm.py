"""RMSNorm fused into the activation quantization (bl_rmsnorm_quantize_act)
against the oracle ("ultragraph -- when the graph is the 1-bit LLM, part 2",
section "attention, as graph ops"; the pre-norm block of "ultragraph-1bit
0.12.0"): codes and scales bit for bit, including rows whose mean of squares
only an exact sum gets right, rows with a huge dynamic range (squares below
the kernel's fixed-point window), subnormals, constant and zero rows."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu
F32 = np.float32


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run(bl, X, g, en=1e-5, eq=1e-5):
    Xq, s = bl.rmsnorm_quantize_act(dev(X), dev(g), en, eq)
    assert bl.sync_status() == "BL_OK"
    rq, rs = oracle.rmsnorm_act_quant(X, g, en, eq)
    np.testing.assert_array_equal(s.cpu().numpy(), rs)
    np.testing.assert_array_equal(Xq.cpu().numpy(), rq)


@pytest.mark.parametrize("M,K", [(1, 2560), (7, 6912), (64, 128), (3, 1001), (2, 3), (1, 1), (300, 512),
                                 (2, 49152)])
def test_random_rows(bl, M, K):
    rng = np.random.default_rng(M * 7 + K)
    X = (rng.standard_normal((M, K)) * rng.uniform(1e-3, 1e3, (M, 1))).astype(F32)
    g = rng.uniform(0.5, 1.5, K).astype(F32) * np.where(rng.random(K) < 0.1, F32(-1), F32(1))
    run(bl, X, g)


def test_exact_mean_of_squares(bl):
    d = 4097
    X = np.full((2, d), F32(2.0 ** -12))
    X[:, 0] = 1.0
    X[1] *= F32(3.0)
    run(bl, X, np.ones(d, F32), 1e-6, 1e-5)


def test_dynamic_range_and_subnormals(bl):
    rng = np.random.default_rng(5)
    X = rng.standard_normal((6, 3000)).astype(F32)
    X[0, ::3] *= F32(2.0 ** -80)           # squares far below the window: exact bins
    X[1, ::5] = F32(1e-42)                 # subnormals
    X[2] *= F32(2.0 ** 60)                 # large magnitudes
    X[3] *= F32(2.0 ** -70)                # the whole row tiny (window below 2^-298 units)
    X[4, 1:] = F32(2.0 ** -100)            # one large value, the rest tiny
    X[5] = F32(1e-45)                      # only the smallest subnormal
    run(bl, X, np.linspace(0.5, 2, 3000, dtype=F32))


def test_constant_zero_and_one_hot_rows(bl):
    K = 1024
    X = np.zeros((4, K), F32)
    X[0] = 2.0
    X[1] = -0.1
    X[3, 17] = 5.0
    g = np.ones(K, F32)
    g[::2] = -1.0
    run(bl, X, g, 2.0 ** -22, 1e-5)


def test_norm_then_linear_matches_oracle(bl):
    """The fused norm's codes and scales drive the integer product: acc from
    bl_linear_acc, dequantized, equals the oracle's layer on RMSNorm(x)."""
    from workloads import random_problem
    p = random_problem(11, 5, 2560, 300)
    g = np.random.default_rng(1).uniform(0.8, 1.2, 2560).astype(F32)
    Xq, s = bl.rmsnorm_quantize_act(dev(p.X), dev(g), 1e-6, p.eps)
    Wp, beta = bl.quantize_weights_pack5(dev(p.W), p.eps)
    acc = bl.linear_acc(Xq, Wp, bl.PACK5, p.N, p.K)
    assert bl.sync_status() == "BL_OK"
    Y = oracle.dequant(acc.cpu().numpy(), s.cpu().numpy(), beta.cpu().numpy()[0])
    ref = oracle.bitlinear(oracle.rmsnorm(p.X, g, 1e-6), p.W, p.eps)["Y"]
    np.testing.assert_array_equal(Y, ref)
