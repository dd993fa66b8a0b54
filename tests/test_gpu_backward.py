"""The straight-through backward (bl_linear_backward) against the float64
oracle ("ultragraph -- when the graph is the 1-bit LLM, part 2", section
"autograd on a byte-graph, and the straight-through lie").

Tolerance, from the arithmetic: every float32 operand is split into two tf32
parts and each product is taken as three tf32 MMAs, so a product is within
3 * 2^-22 |a b| of the exact one; the tensor cores accumulate in float32, at
most n + 1 roundings of 2^-24 relative each (n = 3 * ceil(Kc / 8) accumulator
updates over the contraction length Kc).  So each output must lie within
(3 * 2^-22 + (n + 1) 2^-24) * sum |a b| of the exact sum (the oracle's float64
result, whose own error is far below this).  db is summed in float64 and
rounded once: within 2^-24 |db| + M 2^-53 sum |dY|.
"""
import numpy as np
import pytest

from oracle import backward
from workloads import random_problem

pytestmark = pytest.mark.gpu
F32 = np.float32


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def tol(kc):
    return 3 * 2.0 ** -22 + (3 * -(-kc // 8) + 1) * 2.0 ** -24


def check(got, ref, bound, kc, what):
    err = np.abs(got.astype(np.float64) - ref)
    ratio = float(np.max(err / np.maximum(bound, 1e-300))) if err.size else 0.0
    assert np.all(err <= tol(kc) * bound), f"{what}: max err / sum|ab| = {ratio:.3e} > {tol(kc):.3e}"
    return ratio


@pytest.mark.parametrize("M,N,K", [(8, 256, 128), (2048, 512, 128), (2048, 128, 512), (300, 1000, 700),
                                   (1, 2560, 6912), (129, 257, 33), (5, 3, 1), (777, 2560, 1000)])
def test_backward_against_oracle(bl, M, N, K):
    p = random_problem(M + 3 * N + 7 * K, M, K, N)
    dY = np.random.default_rng(M + N + K).standard_normal((M, N)).astype(F32) * F32(1e-2)
    dX, dW, db = bl.linear_backward(dev(dY), dev(p.X), dev(p.W))
    assert bl.sync_status() == "BL_OK"
    rX, rW, rb = backward.ste_backward(dY, p.X, p.W)
    bX, bW, bb = backward.abs_bound(dY, p.X, p.W)
    rx = check(host(dX), rX, bX, N, "dX")
    rw = check(host(dW), rW, bW, M, "dW")
    err_b = np.abs(host(db).astype(np.float64) - rb)
    assert np.all(err_b <= 2.0 ** -24 * np.abs(rb) + M * 2.0 ** -53 * bb + 1e-300)
    print(f"M={M} N={N} K={K}: max err/sum|ab| dX {rx:.2e} dW {rw:.2e} (tolerance {tol(N):.2e}, {tol(M):.2e})")


def test_backward_large_and_selective(bl):
    """A prefill-sized layer (dW contracts over 4096 rows); dX alone and dW alone
    give the same values as the three together."""
    M, N, K = 4096, 2048, 1024
    rng = np.random.default_rng(9)
    X = rng.standard_normal((M, K), dtype=np.float32)
    W = rng.standard_normal((N, K), dtype=np.float32) * F32(0.02)
    dY = rng.standard_normal((M, N), dtype=np.float32) * F32(1e-3)
    dXd, dWd, dbd = bl.linear_backward(dev(dY), dev(X), dev(W))
    only_x = bl.linear_backward(dev(dY), None, dev(W), want=("dX",))
    only_w = bl.linear_backward(dev(dY), dev(X), None, want=("dW",))
    assert only_x[1] is None and only_x[2] is None and only_w[0] is None
    assert bl.sync_status() == "BL_OK"
    np.testing.assert_array_equal(host(only_x[0]), host(dXd))
    np.testing.assert_array_equal(host(only_w[1]), host(dWd))
    rX, rW, _ = backward.ste_backward(dY, X, W)
    bX, bW, _ = backward.abs_bound(dY, X, W)
    check(host(dXd), rX, bX, N, "dX")
    check(host(dWd), rW, bW, M, "dW")
