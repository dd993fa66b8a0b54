"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Integer outputs (trit codes, packed bytes, int8 codes, int32 accumulators) and
the float32 scales and beta must be bit-exact.  Y must be within 1e-6 relative
error of the oracle (the stated tolerance); since every float step is the same
IEEE operation in the same order, it is also checked to be bit-identical.
"""
import numpy as np
import pytest

import oracle
from workloads import problems, random_problem

pytestmark = pytest.mark.gpu
F32 = np.float32


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


def assert_y_close(y, ref):
    y, ref = np.asarray(y, np.float64), np.asarray(ref, np.float64)
    rel = np.abs(y - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.size == 0 or float(rel.max()) <= 1e-6, f"max rel err {rel.max():.3e}"
    np.testing.assert_array_equal(y, ref)


def check_ok(bl):
    assert bl.sync_status() == "BL_OK"


# ------------------------------------------------------------ weights -------
@pytest.mark.parametrize("N,K", [(256, 128), (7, 3), (1, 1), (33, 81), (300, 2560), (64, 1001)])
def test_quantize_weights_int8(bl, N, K):
    p = random_problem(N * 7 + K, 1, K, N)
    Wq, beta = bl.quantize_weights(dev(p.W), 1e-5)
    rb = oracle.absmean_beta(p.W, 1e-5)
    check_ok(bl)
    assert host(beta)[0] == rb
    np.testing.assert_array_equal(host(Wq), oracle.ternarize(p.W, rb))


@pytest.mark.parametrize("N,K", [(256, 128), (5, 7), (3, 4), (17, 99), (40, 2560), (11, 6912)])
def test_quantize_weights_pack5(bl, N, K):
    p = random_problem(N * 13 + K, 1, K, N)
    Wp, beta = bl.quantize_weights_pack5(dev(p.W), 1e-5)
    rb = oracle.absmean_beta(p.W, 1e-5)
    check_ok(bl)
    assert host(beta)[0] == rb
    np.testing.assert_array_equal(host(Wp), oracle.pack5(oracle.ternarize(p.W, rb)))


def test_beta_wide_dynamic_range(bl):
    """Magnitudes outside the fast accumulator window take the exponent bins."""
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((97, 131)) * 0.02).astype(F32)
    W.ravel()[::7] *= F32(2.0 ** 30)
    W.ravel()[3::11] *= F32(2.0 ** -40)
    W.ravel()[5::13] = F32(1e-42)            # subnormal
    W.ravel()[2::17] = F32(0.0)
    Wq, beta = bl.quantize_weights(dev(W), 1e-5)
    rb = oracle.absmean_beta(W, 1e-5)
    check_ok(bl)
    assert host(beta)[0] == rb
    np.testing.assert_array_equal(host(Wq), oracle.ternarize(W, rb))


def test_beta_constant_tensor_large(bl):
    W = np.full((3001, 1001), F32(0.02), F32)
    _, beta = bl.quantize_weights(dev(W), 1e-5)
    check_ok(bl)
    assert host(beta)[0] == F32(F32(0.02) + F32(1e-5))


def test_ternary_rounding_boundary(bl):
    """Weights placed exactly on, and one float below and above, the place
    where float32(w / beta) crosses 0.5; beta is held fixed by the bulk."""
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((64, 257)) * 0.02).astype(F32)
    for _ in range(3):   # the edits move beta by far less than an ulp; settle it
        b = oracle.absmean_beta(W, 1e-5)
        half = F32(b * F32(0.5))                      # w/beta rounds to 0.5 here
        cand = [half, np.nextafter(half, F32(1)), np.nextafter(half, F32(0)),
                np.nextafter(np.nextafter(half, F32(1)), F32(1))]
        t = F32(b * F32(1.5))
        cand += [t, np.nextafter(t, F32(0)), np.nextafter(t, F32(9))]
        flat = W.ravel()
        for i, c in enumerate(cand):
            flat[10 * i] = c
            flat[10 * i + 1] = -c
    rb = oracle.absmean_beta(W, 1e-5)
    Wq, beta = bl.quantize_weights(dev(W), 1e-5)
    check_ok(bl)
    assert host(beta)[0] == rb
    ref = oracle.ternarize(W, rb)
    np.testing.assert_array_equal(host(Wq), ref)
    assert len(set(ref.ravel()[:80:10].tolist())) > 1   # the boundary really splits


# ------------------------------------------- single-pass weight quantizer ---
# Byte offset of the fix-up mode word in the accumulator block at the start of
# the workspace (after bins[256], four 32-bit counters and slot[256][4]):
# 0 = listed band weights recoded, 1 = whole tensor re-ternarized.
MODE_OFFSET = 256 * 8 + 16 + 256 * 32


def _quantize_single_pass(bl, W, fmt, ws=None):
    N, K = W.shape
    lib = bl.load()
    if ws is None:
        ws = bl.workspace(lib.bl_quantize_weights_workspace_size(N, K), "cuda")
    assert ws.numel() > 16384, "shape should take the single-pass quantizer"
    if fmt == "pack5":
        out, beta = bl.quantize_weights_pack5(dev(W), 1e-5, ws=ws)
    else:
        out, beta = bl.quantize_weights(dev(W), 1e-5, ws=ws)
    mode = int(host(ws[MODE_OFFSET:MODE_OFFSET + 4]).view(np.uint32)[0])
    return host(out), host(beta)[0], mode, ws


def _expect_codes(W, fmt):
    rb = oracle.absmean_beta(W, 1e-5)
    q = oracle.ternarize(W, rb)
    return rb, (oracle.pack5(q) if fmt == "pack5" else q)


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
@pytest.mark.parametrize("N,K", [(512, 2560), (300, 3508), (8000, 132), (262144, 4), (1024, 1040)])
def test_single_pass_gaussian(bl, fmt, N, K):
    """Gaussian weights: the sampled band holds T, so only the band weights are
    recoded (mode 0); chunks of several rows, ragged last groups and pad bytes."""
    p = random_problem(N + 3 * K, 1, K, N)
    out, beta, mode, _ = _quantize_single_pass(bl, p.W, fmt)
    rb, ref = _expect_codes(p.W, fmt)
    check_ok(bl)
    assert beta == rb
    np.testing.assert_array_equal(out, ref)
    assert mode == 0


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
def test_single_pass_wide_range_and_zeros(bl, fmt):
    """Exponent bins, subnormals and exact zeros inside the single pass."""
    rng = np.random.default_rng(15)
    W = (rng.standard_normal((1100, 1000)) * 0.02).astype(F32)
    W.ravel()[::7] *= F32(2.0 ** 30)
    W.ravel()[3::11] *= F32(2.0 ** -40)
    W.ravel()[5::13] = F32(1e-42)
    W.ravel()[2::17] = F32(0.0)
    out, beta, _, _ = _quantize_single_pass(bl, W, fmt)
    rb, ref = _expect_codes(W, fmt)
    check_ok(bl)
    assert beta == rb
    np.testing.assert_array_equal(out, ref)


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
def test_single_pass_band_overflow_falls_back(bl, fmt):
    """Half the magnitudes sit a hair below T (|w| = 1/3 with beta ~ 2/3): the
    band lists overflow and the fix-up re-ternarizes the whole tensor."""
    rng = np.random.default_rng(16)
    mag = np.where(rng.random((1024, 1024)) < 0.5, F32(1.0), F32(1.0 / 3.0)).astype(F32)
    W = (mag * np.where(rng.random(mag.shape) < 0.5, F32(-1), F32(1))).astype(F32)
    out, beta, mode, _ = _quantize_single_pass(bl, W, fmt)
    rb, ref = _expect_codes(W, fmt)
    check_ok(bl)
    assert beta == rb
    np.testing.assert_array_equal(out, ref)
    assert mode == 1


def test_single_pass_unrepresentative_sample_falls_back(bl):
    """Weights shrunk 1000x in every chunk the CTAs read first (chunk i*stride
    mod nch for the first handouts, stride ~ nch/grid and coprime to nch, one
    CTA per SM): the sampled band misses the exact T, and the whole tensor is
    re-ternarized."""
    import math
    import torch
    N, K = 4096, 4096
    p = random_problem(77, 1, K, N)
    W = p.W.copy()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    nch = -(-N * (-(-K // 20)) // 512)
    grid = min(sms, 256, nch)
    stride = max(1, nch // grid)
    while math.gcd(stride, nch) != 1:
        stride += 1
    flat = W.ravel()
    for i in range(3 * grid):          # generous: every early handout
        c = (i * stride) % nch
        g0, g1 = c * 512, min(N * 205, c * 512 + 512)
        r0, r1 = g0 // 205, (g1 - 1) // 205
        f0 = r0 * K + 20 * (g0 - r0 * 205)
        f1 = r1 * K + min(K, 20 * (g1 - 1 - r1 * 205) + 20)
        flat[f0:f1] *= F32(1e-3)
    out, beta, mode, ws = _quantize_single_pass(bl, W, "pack5")
    rb, ref = _expect_codes(W, "pack5")
    check_ok(bl)
    assert beta == rb
    np.testing.assert_array_equal(out, ref)
    assert mode == 1
    # the same workspace again, now with a representative tensor: back to mode 0
    out2, beta2, mode2, _ = _quantize_single_pass(bl, p.W, "pack5", ws=ws)
    rb2, ref2 = _expect_codes(p.W, "pack5")
    check_ok(bl)
    assert beta2 == rb2 and mode2 == 0
    np.testing.assert_array_equal(out2, ref2)


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
def test_single_pass_uncertified_mean_takes_exact_pass(bl, fmt):
    """Half the weights 1.0, half the next float up: the exact mean 1 + 2^-24
    is a float32 rounding tie, so the float64 sum cannot certify beta and the
    kernel adds every magnitude again exactly (ties to even: beta = 1 + eps)."""
    rng = np.random.default_rng(17)
    mag = np.where(rng.permutation(1024 * 1024) < 512 * 1024, F32(1.0),
                   np.nextafter(F32(1.0), F32(2.0))).astype(F32).reshape(1024, 1024)
    W = (mag * np.where(rng.random(mag.shape) < 0.5, F32(-1), F32(1))).astype(F32)
    out, beta, _, _ = _quantize_single_pass(bl, W, fmt)
    rb, ref = _expect_codes(W, fmt)
    check_ok(bl)
    assert rb == F32(F32(1.0) + F32(1e-5))
    assert beta == rb
    np.testing.assert_array_equal(out, ref)


def test_single_pass_nonfinite_is_reported(bl):
    W = random_problem(19, 1, 1024, 1024).W.copy()
    W[700, 33] = np.inf
    _quantize_single_pass(bl, W, "pack5")
    assert bl.sync_status() == "BL_ERR_NONFINITE"
    check_ok(bl)
    # the workspace is clear again: a finite tensor on it is exact
    p = random_problem(20, 1, 1024, 1024)
    lib = bl.load()
    ws = bl.workspace(lib.bl_quantize_weights_workspace_size(1024, 1024), "cuda")
    _quantize_single_pass(bl, W, "pack5", ws=ws)
    assert bl.sync_status() == "BL_ERR_NONFINITE"
    out, beta, _, _ = _quantize_single_pass(bl, p.W, "pack5", ws=ws)
    rb, ref = _expect_codes(p.W, "pack5")
    check_ok(bl)
    assert beta == rb
    np.testing.assert_array_equal(out, ref)


def test_single_pass_workspace_reuse_and_two_pass_agree(bl):
    """The workspace is left clear: repeated calls, and the two-pass kernels on
    the same workspace, give identical results."""
    p = random_problem(91, 1, 2560, 6912)
    lib = bl.load()
    ws = bl.workspace(lib.bl_quantize_weights_workspace_size(6912, 2560), "cuda")
    first = _quantize_single_pass(bl, p.W, "pack5", ws=ws)
    second = _quantize_single_pass(bl, p.W, "pack5", ws=ws)
    Wd = dev(p.W)
    beta = bl.absmean(Wd, 1e-5, ws=ws)
    Wp = host(bl.ternarize_pack5(Wd, beta))
    third = _quantize_single_pass(bl, p.W, "pack5", ws=ws)
    check_ok(bl)
    for r in (second, third):
        assert r[1] == first[1]
        np.testing.assert_array_equal(r[0], first[0])
    assert host(beta)[0] == first[1]
    np.testing.assert_array_equal(Wp, first[0])


# ------------------------------------------------------- the fused forward ---
def _forward_check(bl, X, W, fmt, bias=None, eps=1e-5):
    fmt_c = bl.PACK5 if fmt == "pack5" else bl.I8
    Y, Wd, beta = bl.bitlinear_forward(dev(X), dev(W), fmt_c, None if bias is None else dev(bias), eps)
    ref = oracle.bitlinear(X, W, eps, bias)
    check_ok(bl)
    assert host(beta)[0] == ref["beta"]
    codes = oracle.pack5(ref["Wq"]) if fmt == "pack5" else ref["Wq"]
    np.testing.assert_array_equal(host(Wd), codes)
    assert_y_close(host(Y), ref["Y"])


@pytest.mark.parametrize("fmt", ["pack5", "i8"])
@pytest.mark.parametrize("M,K,N", [(1, 2560, 6912), (1, 6912, 2560), (2, 1040, 1024), (3, 3508, 300),
                                   (4, 132, 8000), (1, 12288, 128)])
def test_forward_one_launch(bl, fmt, M, K, N):
    """M <= 4: weight quantization, activation quantization, contraction and
    dequant in the single pass over W; Y bit-identical to the oracle."""
    p = random_problem(M * 1000 + K + N, M, K, N)
    bias = (np.random.default_rng(M + K).standard_normal(N) * 0.1).astype(F32) if M % 2 else None
    _forward_check(bl, p.X, p.W, fmt, bias)


def test_forward_decode_outliers(bl):
    """The decode workload's activations (1% of entries x20) through the forward."""
    for p in problems(2):
        _forward_check(bl, p.X, p.W, "pack5")


@pytest.mark.parametrize("fmt", ["pack5", "i8"])
def test_forward_band_overflow_corrects_sums(bl, fmt):
    """Mode 1 (every group re-coded): the row sums get every group's correction."""
    rng = np.random.default_rng(21)
    mag = np.where(rng.random((1024, 1024)) < 0.5, F32(1.0), F32(1.0 / 3.0)).astype(F32)
    W = (mag * np.where(rng.random(mag.shape) < 0.5, F32(-1), F32(1))).astype(F32)
    X = rng.standard_normal((2, 1024)).astype(F32)
    _forward_check(bl, X, W, fmt)


def test_forward_uncertified_mean(bl):
    """The float32 rounding tie of beta (exact pass) inside the forward."""
    rng = np.random.default_rng(22)
    mag = np.where(rng.permutation(1024 * 1024) < 512 * 1024, F32(1.0),
                   np.nextafter(F32(1.0), F32(2.0))).astype(F32).reshape(1024, 1024)
    W = (mag * np.where(rng.random(mag.shape) < 0.5, F32(-1), F32(1))).astype(F32)
    X = rng.standard_normal((1, 1024)).astype(F32)
    _forward_check(bl, X, W, "pack5")


@pytest.mark.parametrize("M,K,N", [(5, 1040, 1024), (1, 1001, 1100), (64, 256, 256), (1, 40, 30)])
def test_forward_two_call_shapes(bl, M, K, N):
    """Shapes outside the one-launch path (M > 4, K % 4 != 0, small tensors)."""
    p = random_problem(M + K + N + 7, M, K, N)
    _forward_check(bl, p.X, p.W, "pack5")
    _forward_check(bl, p.X, p.W, "i8")


def test_forward_repeat_same_workspace(bl):
    p = random_problem(23, 1, 2560, 6912)
    lib = bl.load()
    ws = bl.workspace(lib.bl_bitlinear_forward_workspace_size(1, 6912, 2560, bl.PACK5), "cuda")
    outs = [host(bl.bitlinear_forward(dev(p.X), dev(p.W), bl.PACK5, ws=ws)[0]) for _ in range(3)]
    check_ok(bl)
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])
    assert_y_close(outs[0], oracle.bitlinear(p.X, p.W, 1e-5)["Y"])


def test_nonfinite_weight_is_reported(bl):
    W = np.ones((4, 8), F32)
    W[2, 3] = np.inf
    bl.quantize_weights(dev(W), 1e-5)
    assert bl.sync_status() == "BL_ERR_NONFINITE"
    check_ok(bl)


# ------------------------------------------------------------ packing -------
@pytest.mark.parametrize("N,K", [(1, 1), (3, 5), (7, 23), (64, 2560), (9, 6913)])
def test_pack_unpack(bl, N, K):
    rng = np.random.default_rng(K)
    Wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
    Wp = bl.pack(dev(Wq))
    np.testing.assert_array_equal(host(Wp), oracle.pack5(Wq))
    np.testing.assert_array_equal(host(bl.unpack(Wp, K)), Wq)
    check_ok(bl)


def test_pack_all_patterns(bl):
    import itertools
    pats = np.array(list(itertools.product((-1, 0, 1), repeat=5)), np.int8).reshape(1, -1)
    Wp = bl.pack(dev(pats))
    np.testing.assert_array_equal(host(Wp), oracle.pack5(pats))


# ------------------------------------------------------------ activations ---
@pytest.mark.parametrize("M,K", [(8, 128), (1, 2560), (3, 7), (5, 1), (17, 6912), (2, 11008), (70, 333),
                                 (9, 8192), (3, 12288), (4, 16384), (3, 30000), (2, 32768), (2, 40000)])
def test_quantize_act(bl, M, K):
    p = random_problem(M * 3 + K, M, K, 1)
    X = p.X * np.linspace(0.01, 100, M, dtype=F32)[:, None]
    Xq, s = bl.quantize_act(dev(X), 1e-5)
    rq, rs = oracle.act_quant(X, 1e-5)
    check_ok(bl)
    np.testing.assert_array_equal(host(s), rs)
    np.testing.assert_array_equal(host(Xq), rq)


@pytest.mark.parametrize("M,K", [(600, 4096), (700, 1000), (320, 12288), (1000, 12), (297, 16384), (4096, 4),
                                 (1203, 11008), (400, 16388)])
def test_quantize_act_many_rows(bl, M, K):
    """Many rows, one CTA per row (the register kernel up to K = 16384, the
    two-pass kernel beyond, and for rows that are not whole float4s); codes and
    scales as the oracle's."""
    rng = np.random.default_rng(M + K)
    X = rng.standard_normal((M, K)).astype(F32)
    X[::17] *= F32(40.0)
    X[5] = 0.0
    Xq, s = bl.quantize_act(dev(X), 1e-5)
    rq, rs = oracle.act_quant(X, 1e-5)
    check_ok(bl)
    np.testing.assert_array_equal(host(s), rs)
    np.testing.assert_array_equal(host(Xq), rq)


def test_quantize_act_ties_and_zero_rows(bl):
    X = np.zeros((4, 9), F32)
    X[0] = [127, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 126.5, -127]
    X[2] = [-127, 63.5, 0, 1, 2, 3, 4, 5, 6]
    for eps in (2.0 ** -30, 1e-5, 2.0 ** -10):
        Xq, s = bl.quantize_act(dev(X), eps)
        rq, rs = oracle.act_quant(X, eps)
        np.testing.assert_array_equal(host(s), rs)
        np.testing.assert_array_equal(host(Xq), rq)
    check_ok(bl)


@pytest.mark.parametrize("M", [1, 3, 4, 9])
def test_near_tie_groups_in_fused_quantization(bl, M):
    """Quotients within the fast path's 2^-15 window of a half-integer, placed in
    the 20-activation groups that the GEMV (M <= 3) and the swapped GEMM's
    quantizer (M >= 4) code together: one such element in a group (the single
    exact division on the hot path), two in a group, and one in the ragged last
    group.  Codes, scales and Y must equal the oracle's."""
    rng = np.random.default_rng(21)
    K, N = 413, 96
    X = rng.standard_normal((M, K)).astype(F32)
    X[:, 0] = 100.0                                    # fixes max|x| per row
    eps = F32(1e-5)
    s = (F32(100.0) / F32(127)).astype(F32) + eps      # the scale every row gets
    for m in range(M):
        for k, h in ((3, 2.5), (25, -7.5), (31, 11.5), (410, 0.5)):   # group 0: one; group 1: two; last group
            X[m, k] = F32(h) * s
    p = random_problem(5, M, K, N)
    Wd, beta = bl.quantize_weights_pack5(dev(p.W), p.eps)
    ref = oracle.bitlinear(X, p.W, eps)["Y"]
    rq, _ = oracle.act_quant(X, eps)
    assert any(abs(float(X[0, k]) / float(s) - h) < 2.0 ** -15 for k, h in ((3, 2.5),))
    Y = bl.linear(dev(X), Wd, bl.PACK5, N, K, beta, eps=float(eps))
    check_ok(bl)
    assert_y_close(host(Y), ref)
    Xq, _ = bl.quantize_act(dev(X), float(eps))
    np.testing.assert_array_equal(host(Xq), rq)


@pytest.mark.parametrize("M", [1, 2, 5])
def test_many_near_ties_in_fused_quantization(bl, M):
    """Every 5-activation unit (a quarter of a 20-activation group) holds one
    product within the fast path's window
    of a half-integer (quotients a few ulps either side of n + 1/2,
    n = 0..125, both signs), every seventh unit a second one: the division-free exact code
    and the per-element fallback against the oracle's float32 division."""
    rng = np.random.default_rng(22)
    K, N = 2000, 64
    X = rng.standard_normal((M, K)).astype(F32)
    X[:, 0] = 127.0
    eps = F32(2.0 ** -12)
    s = (F32(127.0) / F32(127)).astype(F32) + eps
    for m in range(M):
        for u in range(1, K // 5):
            for k in ([5 * u + 1] + ([5 * u + 3] if u % 7 == 0 else [])):
                h = F32(int(rng.integers(0, 126)) + 0.5)     # |x| stays below the row max 127
                x = F32(h * s)
                for _ in range(int(rng.integers(0, 6))):
                    x = np.nextafter(x, F32(np.inf) if rng.integers(0, 2) else F32(-np.inf)).astype(F32)
                X[m, k] = x if rng.integers(0, 2) else -x
    p = random_problem(6, M, K, N)
    Wd, beta = bl.quantize_weights_pack5(dev(p.W), float(eps))      # the oracle uses one eps for both
    Y = bl.linear(dev(X), Wd, bl.PACK5, N, K, beta, eps=float(eps))
    check_ok(bl)
    assert_y_close(host(Y), oracle.bitlinear(X, p.W, eps)["Y"])


def test_nonfinite_activation_is_reported(bl):
    X = np.ones((3, 10), F32)
    X[1, 4] = np.nan
    bl.quantize_act(dev(X), 1e-5)
    assert bl.sync_status() == "BL_ERR_NONFINITE"
    check_ok(bl)


# ------------------------------------------------------------ linear --------
def _layer(bl, p, fmt, path, bias=None):
    if fmt == bl.PACK5:
        Wd, beta = bl.quantize_weights_pack5(dev(p.W), p.eps)
    else:
        Wd, beta = bl.quantize_weights(dev(p.W), p.eps)
    Y = bl.linear(dev(p.X), Wd, fmt, p.N, p.K, beta, None if bias is None else dev(bias),
                  p.eps, path=path)
    return host(Y), Wd, beta


PATHS = ["simt", "gemv", "tc", "auto"]


def _path(bl, name):
    return {"simt": bl.PATH_SIMT, "auto": bl.PATH_AUTO, "gemv": bl.PATH_GEMV,
            "tc": bl.PATH_TC}[name]


@pytest.mark.parametrize("path", PATHS)
@pytest.mark.parametrize("fmt", ["i8", "pack5"])
@pytest.mark.parametrize("M,K,N", [(8, 128, 256), (1, 2560, 96), (3, 7, 5), (65, 161, 130),
                                   (130, 1001, 67), (2, 6912, 40), (1, 1, 1)])
def test_linear_small(bl, path, fmt, M, K, N):
    p = random_problem(M + 10 * K + 100 * N, M, K, N)
    f = bl.PACK5 if fmt == "pack5" else bl.I8
    if bl.linear_plan(M, N, K, f, _path(bl, path))[0] < 0:
        with pytest.raises(bl.BitLinearError) as e:
            _layer(bl, p, f, _path(bl, path))
        assert e.value.status == "BL_ERR_UNSUPPORTED"
        return
    Y, _, _ = _layer(bl, p, f, _path(bl, path))
    check_ok(bl)
    assert_y_close(Y, oracle.bitlinear(p.X, p.W, p.eps)["Y"])


@pytest.mark.parametrize("M,K,N", [
    (1, 2560, 6912), (1, 6912, 2560), (2, 2560, 300), (3, 999, 149), (4, 2560, 1000),
    (1, 11008, 2000),       # K split over two warp slices
    (4, 11008, 2000),       # four rows, five slices
    (2, 8192, 777), (4, 8192, 148), (1, 5, 3), (4, 1, 1),
    (1, 81, 40000)])        # 271 rows per CTA in 1 KB stages: the ring of 8 is reused
def test_gemv_parity(bl, M, K, N):
    assert bl.linear_plan(M, N, K, bl.PACK5, bl.PATH_GEMV)[0] == bl.PATH_GEMV
    p = random_problem(3 * M + K + N, M, K, N)
    Y, Wd, beta = _layer(bl, p, bl.PACK5, bl.PATH_GEMV)
    check_ok(bl)
    assert_y_close(Y, oracle.bitlinear(p.X, p.W, p.eps)["Y"])
    Xq, s = oracle.act_quant(p.X, p.eps)
    acc = bl.linear_acc(dev(Xq), Wd, bl.PACK5, N, K, path=bl.PATH_GEMV)
    check_ok(bl)
    np.testing.assert_array_equal(host(acc), oracle.contract(Xq, oracle.ternarize(p.W, host(beta)[0])))


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
@pytest.mark.parametrize("M,K,N", [(128, 128, 256), (256, 4096, 512), (300, 1000, 1000),
                                   (129, 2560, 257), (512, 640, 96), (4, 384, 600)])
def test_tc_parity(bl, fmt, M, K, N):
    """tcgen05 GEMM: one or several 128 x 256 tiles, ragged M, N and K tails."""
    f = bl.PACK5 if fmt == "pack5" else bl.I8
    p = random_problem(7 * M + K + N, M, K, N)
    b = np.random.default_rng(M).standard_normal(N).astype(F32)
    if f == bl.I8 and K % 16:          # contiguous int8 rows of K bytes: not TMA-aligned
        assert bl.linear_plan(M, N, K, f, bl.PATH_TC)[0] == -1
        with pytest.raises(bl.BitLinearError) as e:
            _layer(bl, p, f, bl.PATH_TC, bias=b)
        assert e.value.status == "BL_ERR_UNSUPPORTED"
        return
    assert bl.linear_plan(M, N, K, f, bl.PATH_TC)[0] == bl.PATH_TC
    Y, Wd, beta = _layer(bl, p, f, bl.PATH_TC, bias=b)
    check_ok(bl)
    assert_y_close(Y, oracle.bitlinear(p.X, p.W, p.eps, bias=b)["Y"])
    if K % 16 == 0:
        Xq, s = oracle.act_quant(p.X, p.eps)
        acc = bl.linear_acc(dev(Xq), Wd, f, N, K, path=bl.PATH_TC)
        check_ok(bl)
        np.testing.assert_array_equal(host(acc), oracle.contract(Xq, oracle.ternarize(p.W, host(beta)[0])))


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
@pytest.mark.parametrize("M,K,N", [(5, 6912, 2560), (40, 2560, 6912), (127, 1040, 1000), (9, 128, 70)])
def test_small_m_tensor_core_auto(bl, fmt, M, K, N):
    """5 <= M < 128 with AUTO: the tcgen05 GEMM with K split across CTAs (few
    128 x 256 tiles), the partials summed by the reduction kernel; ragged N
    tails inside a tile."""
    f = bl.PACK5 if fmt == "pack5" else bl.I8
    assert bl.linear_plan(M, N, K, f, bl.PATH_AUTO)[0] == bl.PATH_TC
    p = random_problem(M * 31 + K + N, M, K, N)
    Y, Wd, beta = _layer(bl, p, f, bl.PATH_AUTO)
    ref = oracle.bitlinear(p.X, p.W, p.eps)
    check_ok(bl)
    assert_y_close(Y, ref["Y"])


@pytest.mark.parametrize("M,K,N", [(385, 1300, 9500), (129, 700, 19000), (640, 1040, 300)])
def test_tc_packed_routes(bl, M, K, N):
    """Packed weights on the tensor cores, both routes: decoded inside the GEMM
    for up to 4 row tiles of 128 (the first two shapes fill the SMs without a K
    split, and K ends inside a 640-trit chunk), unpacked to int8 once beyond
    that (the third, whose K is also split in two)."""
    p = random_problem(M + 3 * K + 7 * N, M, K, N)
    path, n = bl.linear_plan(M, N, K, bl.PACK5, bl.PATH_AUTO)
    # act_quant + GEMM, + unpack beyond 4 row tiles, + the K-split reduction
    # when there are fewer 128 x 256 tiles than half of 148 SMs (and K has at
    # least two 640-wide chunks)
    tiles = -(-M // 128) * -(-N // 256)
    chunks = -(-(-(-K // 128)) // 5)
    split = min(148 // tiles, chunks, 8)
    assert path == bl.PATH_TC and n == 2 + (M > 4 * 128) + (split > 1)
    _sampled_check(bl, p, bl.PACK5, n_samples=4096, seed=M)


def test_linear_acc_without_workspace_decodes_in_the_gemm(bl):
    """bl_linear_acc takes no workspace: at M = 640 (5 row tiles) with packed
    weights the tensor-core GEMM then decodes the trits itself instead of
    reading an unpacked copy, and K is not split; acc must equal the exact
    contraction."""
    import torch
    M, K, N = 640, 1040, 300
    p = random_problem(M + K + N + 5, M, K, N)
    Wd, beta = bl.quantize_weights_pack5(dev(p.W), p.eps)
    Xq, _ = oracle.act_quant(p.X, p.eps)
    Xd = dev(Xq)
    acc = torch.empty((M, N), dtype=torch.int32, device="cuda")
    st = bl.load().bl_linear_acc(Xd.data_ptr(), M, K, Wd.data_ptr(), bl.PACK5, N, Wd.shape[1],
                                 acc.data_ptr(), None)
    assert bl.STATUS[st] == "BL_OK"
    check_ok(bl)
    np.testing.assert_array_equal(host(acc), oracle.contract(Xq, oracle.ternarize(p.W, host(beta)[0])))


def test_linear_bias(bl):
    p = random_problem(77, 5, 300, 45)
    b = np.random.default_rng(1).standard_normal(45).astype(F32)
    Y, _, _ = _layer(bl, p, bl.PACK5, bl.PATH_AUTO, bias=b)
    check_ok(bl)
    assert_y_close(Y, oracle.bitlinear(p.X, p.W, p.eps, bias=b)["Y"])


def acc_supported(bl, M, N, K, f, path):
    """Whether bl_linear_acc_ex takes the pinned path with contiguous X_q [M, K]."""
    if path == bl.PATH_TC:
        # the swapped GEMM (packed weights, M <= 128) reads a decode-order copy of
        # X_q in the workspace; otherwise X_q rows of K bytes must be TMA-aligned
        swapped = f == bl.PACK5 and M <= 128
        return K >= 128 and (swapped or K % 16 == 0) and bl.linear_plan(M, N, K, f, path)[0] == path
    return bl.linear_plan(M, N, K, f, path)[0] == path or path == bl.PATH_AUTO


@pytest.mark.parametrize("K", [517, 528])
@pytest.mark.parametrize("path", PATHS)
def test_linear_acc_exact(bl, path, K):
    rng = np.random.default_rng(3)
    M, N = 37, 71
    p = _path(bl, path)
    Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    Wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
    for m in (M, 1, 2, 4):     # 1..4: the GEMV's row counts
        ref = oracle.contract(Xq[:m], Wq)
        for f, Wd in ((bl.I8, dev(Wq)), (bl.PACK5, bl.pack(dev(Wq)))):
            if not acc_supported(bl, m, N, K, f, p):
                with pytest.raises(bl.BitLinearError) as e:
                    bl.linear_acc(dev(Xq[:m]), Wd, f, N, K, path=p)
                assert e.value.status == "BL_ERR_UNSUPPORTED"
                continue
            acc = bl.linear_acc(dev(Xq[:m]), Wd, f, N, K, path=p)
            check_ok(bl)
            np.testing.assert_array_equal(host(acc), ref)


def test_linear_extreme_accumulators(bl):
    K = 8192
    Xq = np.full((2, K), 127, np.int8)
    Xq[1] = -127
    Wq = np.ones((3, K), np.int8)
    Wq[1] = -1
    Wq[2, ::2] = 0
    acc = bl.linear_acc(dev(Xq), bl.pack(dev(Wq)), bl.PACK5, 3, K)
    check_ok(bl)
    np.testing.assert_array_equal(host(acc), oracle.contract(Xq, Wq))


def test_workload_tiny(bl):
    p = next(problems(1))
    Y, Wd, beta = _layer(bl, p, bl.I8, bl.PATH_AUTO)
    r = oracle.bitlinear(p.X, p.W, p.eps)
    check_ok(bl)
    assert host(beta)[0] == r["beta"]
    np.testing.assert_array_equal(host(Wd), r["Wq"])
    assert_y_close(Y, r["Y"])


def test_workload_gpt_layers(bl):
    """All 24 BitLinears of the d_model-128, 4-layer ternary GPT at M = 2048."""
    for p in problems(3):
        Y, _, _ = _layer(bl, p, bl.I8, bl.PATH_AUTO)
        assert_y_close(Y, oracle.bitlinear(p.X, p.W, p.eps)["Y"])
    check_ok(bl)


def test_row_independence_and_batching(bl):
    """Per-token scales: a row's output is the same alone or in a batch, and
    does not move when another row changes ("attention, as graph ops")."""
    p = random_problem(9, 12, 700, 50)
    Wp, beta = bl.quantize_weights_pack5(dev(p.W), p.eps)
    Y = host(bl.linear(dev(p.X), Wp, bl.PACK5, p.N, p.K, beta))
    for m in (0, 5, 11):
        one = host(bl.linear(dev(p.X[m:m + 1]), Wp, bl.PACK5, p.N, p.K, beta))
        np.testing.assert_array_equal(one[0], Y[m])
    X2 = p.X.copy()
    X2[3] *= F32(1e4)
    Y2 = host(bl.linear(dev(X2), Wp, bl.PACK5, p.N, p.K, beta))
    keep = [r for r in range(12) if r != 3]
    np.testing.assert_array_equal(Y2[keep], Y[keep])
    check_ok(bl)


def test_repeatable(bl):
    p = random_problem(10, 33, 999, 77)
    a, _, _ = _layer(bl, p, bl.PACK5, bl.PATH_AUTO)
    b, _, _ = _layer(bl, p, bl.PACK5, bl.PATH_AUTO)
    np.testing.assert_array_equal(a, b)


# ------------------------------------------------ full sizes, sampled ------
_PROBLEM_CACHE = {}
_BETA_CACHE = {}


def _problem(wid, idx):
    key = (wid, idx)
    if key not in _PROBLEM_CACHE:
        if wid == 5 and _PROBLEM_CACHE:       # keep one shared 8192^2 weight, not ten
            for k in [k for k in _PROBLEM_CACHE if k[0] != 5]:
                del _PROBLEM_CACHE[k]
        if wid == 5:
            for i, p in enumerate(problems(5)):
                _PROBLEM_CACHE[(5, i)] = p
        else:
            _PROBLEM_CACHE.clear()
            _PROBLEM_CACHE[key] = next(problems(wid, only=[idx]))
    return _PROBLEM_CACHE[key]


def _oracle_beta(p):
    key = (p.workload, id(p.W))
    if key not in _BETA_CACHE:
        _BETA_CACHE.clear()
        _BETA_CACHE[key] = oracle.absmean_beta(p.W, p.eps)
    return _BETA_CACHE[key]


def _sampled_check(bl, p, fmt, n_samples=512, seed=0):
    """Full-size call on the GPU; the oracle computes sampled outputs one by one
    (beta over the whole tensor, row quantization for the sampled rows only)."""
    import torch
    Wd_fn = bl.quantize_weights_pack5 if fmt == bl.PACK5 else bl.quantize_weights
    Wd, beta = Wd_fn(dev(p.W), p.eps)
    Y = bl.linear(dev(p.X), Wd, fmt, p.N, p.K, beta, eps=p.eps)
    torch.cuda.synchronize()
    check_ok(bl)
    rb = _oracle_beta(p)
    assert host(beta)[0] == rb
    rng = np.random.default_rng(seed)
    ms = rng.integers(0, p.M, n_samples)
    ns = rng.integers(0, p.N, n_samples)
    ms[:2], ns[:2] = [0, p.M - 1], [p.N - 1, 0]
    Xq, s = oracle.act_quant(p.X[ms], p.eps)
    Wq = oracle.ternarize(p.W[ns], rb)
    acc = oracle.contract_entries(Xq, Wq)
    ref = oracle.dequant(acc, s, rb)
    got = host(Y)[ms, ns]
    assert_y_close(got, ref)
    rows = np.unique(ns)[:64]
    if fmt == bl.PACK5:
        np.testing.assert_array_equal(host(Wd)[rows], oracle.pack5(oracle.ternarize(p.W[rows], rb)))
    else:
        np.testing.assert_array_equal(host(Wd)[rows], oracle.ternarize(p.W[rows], rb))


@pytest.mark.parametrize("idx", [0, 1])
def test_workload_decode_full(bl, idx):
    p = _problem(2, idx)
    _sampled_check(bl, p, bl.PACK5, n_samples=p.N)   # M = 1: every output


@pytest.mark.parametrize("idx", [0, 1])
def test_workload_prefill_full_sampled(bl, idx):
    p = _problem(4, idx)
    _sampled_check(bl, p, bl.PACK5, n_samples=512, seed=idx)


@pytest.mark.parametrize("idx", range(10))
def test_workload_sweep_full_sampled(bl, idx):
    p = _problem(5, idx)
    _sampled_check(bl, p, bl.PACK5, n_samples=256, seed=idx)
