"""bl_linear_noalloc: the BitLinear forward for callers that cannot allocate
device memory (plugin / custom-op interfaces that own every allocation, or
loops where a cudaMalloc that may synchronize the device is not allowed).

It is called here through the C ABI and must give the same Y as the existing
bl_linear entry point, within the 1e-6 relative tolerance the other parity tests
use, on two calls in a row (the shared static scratch keeps the previous call's
contents, which must not leak into the next result).  This file is collected
last so a run that stops at the first failure has already run everything else.
"""
import ctypes

import numpy as np
import pytest

from workloads import random_problem

pytestmark = pytest.mark.gpu


def _noalloc(bl, X, W, fmt, N, K, beta, Y, eps):
    import torch
    lib = bl.load()
    return lib.bl_linear_noalloc(X.data_ptr(), X.shape[0], K, W.data_ptr(), fmt, N, W.shape[1],
                                 beta.data_ptr(), None, eps, Y.data_ptr(),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    rel = np.abs(a - b) / np.maximum(np.abs(b), 1e-30)
    assert float(rel.max()) <= 1e-6, f"max rel err {rel.max():.3e}"


@pytest.mark.parametrize("fmt_name,M,K,N", [("pack5", 1, 2560, 6912), ("pack5", 37, 1001, 67),
                                            ("i8", 8, 128, 256)])
def test_noalloc_matches_bl_linear_twice(bl, fmt_name, M, K, N):
    import torch
    fmt = bl.PACK5 if fmt_name == "pack5" else bl.I8
    p = random_problem(M * 31 + K + N, M, K, N)
    W = torch.from_numpy(p.W).cuda()
    Wd, beta = (bl.quantize_weights_pack5(W, p.eps) if fmt == bl.PACK5
                else bl.quantize_weights(W, p.eps))
    rng = np.random.default_rng(7)
    for call in range(2):   # second call: different activations, same scratch
        X = torch.from_numpy((p.X * np.float32(1 + 3 * call) +
                              rng.standard_normal(p.X.shape).astype(np.float32))).cuda()
        ref = bl.linear(X, Wd, fmt, N, K, beta, eps=p.eps)
        Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(bl, X, Wd, fmt, N, K, beta, Y, p.eps) == 0
        assert bl.sync_status() == "BL_OK"
        _close(Y.cpu().numpy(), ref.cpu().numpy())


def test_noalloc_rejects_shapes_beyond_its_scratch(bl):
    import torch
    K = 4096
    M = bl.NOALLOC_SCRATCH_BYTES // K + 1           # quantized X alone no longer fits
    lib = bl.load()
    assert lib.bl_linear_workspace_size(M, 16, K, bl.PACK5) > bl.NOALLOC_SCRATCH_BYTES
    W = torch.zeros((16, bl.pack5_ldp(K)), dtype=torch.uint8, device="cuda")
    beta = torch.ones(1, dtype=torch.float32, device="cuda")
    X = torch.zeros((1, K), dtype=torch.float32, device="cuda")   # never read
    Y = torch.zeros((1, 16), dtype=torch.float32, device="cuda")
    code = lib.bl_linear_noalloc(X.data_ptr(), M, K, W.data_ptr(), bl.PACK5, 16, W.shape[1],
                                 beta.data_ptr(), None, 1e-5, Y.data_ptr(), None)
    assert bl.STATUS[code] == "BL_ERR_WORKSPACE"


def test_noalloc_drops_the_k_split_when_its_partials_do_not_fit(bl):
    """M = 512, K = 11008, N = 4096 on the tensor cores: 64 tiles of 128 x 256, so
    bl_linear splits K in two and its workspace (5.6 MB of X_q + 16.8 MB of
    int32 partials) exceeds the 16 MB array; bl_linear_noalloc runs the GEMM
    unsplit instead and must give the same Y (integer sums are exact)."""
    import torch
    M, K, N = 512, 11008, 4096
    lib = bl.load()
    assert lib.bl_linear_workspace_size(M, N, K, bl.PACK5) > bl.NOALLOC_SCRATCH_BYTES
    rng = np.random.default_rng(11)
    Wh = rng.standard_normal((N, K), dtype=np.float32) * np.float32(0.02)
    Xh = rng.standard_normal((M, K), dtype=np.float32)
    Wd, beta = bl.quantize_weights_pack5(torch.from_numpy(Wh).cuda(), 1e-5)
    X = torch.from_numpy(Xh).cuda()
    ref = bl.linear(X, Wd, bl.PACK5, N, K, beta, eps=1e-5)
    Y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    assert _noalloc(bl, X, Wd, bl.PACK5, N, K, beta, Y, 1e-5) == 0
    assert bl.sync_status() == "BL_OK"
    got = Y.cpu().numpy()
    np.testing.assert_array_equal(got, ref.cpu().numpy())
    # and every element against the oracle itself
    import oracle
    rb = oracle.absmean_beta(Wh, 1e-5)
    assert beta.cpu().numpy()[0] == rb
    Xq, s = oracle.act_quant(Xh, 1e-5)
    acc = oracle.contract_f64(Xq, oracle.ternarize(Wh, rb))
    np.testing.assert_array_equal(got, oracle.dequant(acc, s, rb))
