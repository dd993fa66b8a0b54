"""The decode GEMV's launch modes against the oracle: several problems in one
launch (bl_linear_group), weights streamed before the dependency wait
(BL_FLAG_STATIC_WEIGHTS), and back-to-back launches that overlap through
programmatic dependent launch -- including chains whose next input is the
previous output, and weights rewritten by the kernel right before the GEMV.
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


def assert_y_exact(y, ref):
    y, ref = np.asarray(y, np.float64), np.asarray(ref, np.float64)
    rel = np.abs(y - ref) / np.maximum(np.abs(ref), 1e-30)
    assert rel.size == 0 or float(rel.max()) <= 1e-6, f"max rel err {rel.max():.3e}"
    np.testing.assert_array_equal(y, ref)


class _P:
    """A weight tensor alone, as the quantization helper takes it."""
    def __init__(self, W):
        self.W, self.eps = W, 1e-5


def quantized(bl, p, fmt=None):
    fmt = bl.PACK5 if fmt is None else fmt
    fn = bl.quantize_weights_pack5 if fmt == bl.PACK5 else bl.quantize_weights
    return fn(dev(p.W), p.eps)


@pytest.mark.parametrize("static", [False, True])
def test_group_decode_workload(bl, static):
    """Both decode-workload layers in one launch, every output against the oracle."""
    ps = list(problems(2))
    calls, refs = [], []
    for p in ps:
        Wd, beta = quantized(bl, p)
        calls.append((dev(p.X), Wd, bl.PACK5, p.N, p.K, beta, None, p.eps))
        refs.append(oracle.bitlinear(p.X, p.W, p.eps)["Y"])
    lib = bl.load()
    arr = (bl.LinearCall * 2)()
    for i, (X, Wd, f, N, K, beta, _, eps) in enumerate(calls):
        arr[i] = bl.LinearCall(X.data_ptr(), 1, K, Wd.data_ptr(), N, Wd.shape[1], f, eps, beta.data_ptr(), None, 0)
    assert lib.bl_linear_group_workspace_size(arr, 2) == 0
    Ys = bl.linear_group(calls, static_weights=static)
    assert bl.sync_status() == "BL_OK"
    for Y, ref in zip(Ys, refs):
        assert_y_exact(host(Y), ref)


def test_group_mixed_calls(bl):
    """Six decode calls (M = 1 and 2, ragged K, bias) -- two launches for M = 1
    (at most four problems each) and one for M = 2 -- beside a tensor-core call
    and a one-trit-per-byte call that take bl_linear's own paths."""
    specs = [(1, 2560, 700), (1, 999, 1500), (1, 6912, 257), (1, 40, 3000), (1, 8192, 64),
             (2, 3000, 500), (64, 1040, 300), (3, 77, 90)]
    calls, refs = [], []
    for i, (M, K, N) in enumerate(specs):
        p = random_problem(900 + i, M, K, N)
        fmt = bl.I8 if i == len(specs) - 1 else bl.PACK5
        Wd, beta = quantized(bl, p, fmt)
        bias = (np.random.default_rng(i).standard_normal(N) * 0.1).astype(F32) if i % 2 else None
        calls.append((dev(p.X), Wd, fmt, N, K, beta, None if bias is None else dev(bias), p.eps))
        refs.append(oracle.bitlinear(p.X, p.W, p.eps, bias)["Y"])
    Ys = bl.linear_group(calls, static_weights=True)
    assert bl.sync_status() == "BL_OK"
    for Y, ref in zip(Ys, refs):
        assert_y_exact(host(Y), ref)


@pytest.mark.parametrize("M,K,N", [(1, 50000, 300), (2, 50000, 200), (2, 20000, 333), (4, 30000, 129),
                                   (3, 12345, 1000)])
def test_gemv_long_rows(bl, M, K, N):
    """Rows of up to 10000 packed bytes: several 16-byte chunks per lane and up
    to 16 warps per row slice (M = 4 at K = 30000: 120 KB of decode-order codes
    beside the 64 KB table)."""
    p = random_problem(M * 7 + K + N, M, K, N)
    Wd, beta = quantized(bl, p)
    assert bl.linear_plan(M, N, K, bl.PACK5, bl.PATH_GEMV)[0] == bl.PATH_GEMV
    for static in (False, True):
        Y = bl.linear(dev(p.X), Wd, bl.PACK5, N, K, beta, eps=p.eps, path=bl.PATH_GEMV, static_weights=static)
        assert bl.sync_status() == "BL_OK"
        assert_y_exact(host(Y), oracle.bitlinear(p.X, p.W, p.eps)["Y"])


def test_gemv_declines_codes_beyond_shared_memory(bl):
    """M = 4 at K = 40000 needs 160 KB of decode-order codes: the GEMV declines
    and AUTO takes another path (the answer is the same)."""
    assert bl.linear_plan(4, 129, 40000, bl.PACK5, bl.PATH_GEMV)[0] == -1
    assert bl.linear_plan(4, 129, 40000, bl.PACK5)[0] == bl.PATH_TC
    p = random_problem(77, 4, 40000, 129)
    Wd, beta = quantized(bl, p)
    Y = bl.linear(dev(p.X), Wd, bl.PACK5, 129, 40000, beta, eps=p.eps)
    assert bl.sync_status() == "BL_OK"
    assert_y_exact(host(Y), oracle.bitlinear(p.X, p.W, p.eps)["Y"])


@pytest.mark.parametrize("M", [1, 2])
def test_gemv_segment_ring(bl, M):
    """K = 6912, N = 16000: each CTA's 109 rows of packed weights (152 KB) do not
    fit its shared memory at once, so they stream through a ring of segments
    reused as the CTA computes.  Every output against the oracle (weights
    ternarized and contracted in row blocks to bound host memory)."""
    K, N, eps = 6912, 16000, 1e-5
    rng = np.random.default_rng(31 + M)
    W = rng.standard_normal((N, K), dtype=np.float32) * F32(0.02)
    X = rng.standard_normal((M, K), dtype=np.float32)
    Wd, beta = quantized(bl, _P(W))
    Y = host(bl.linear(dev(X), Wd, bl.PACK5, N, K, beta, eps=eps, path=bl.PATH_GEMV))
    assert bl.sync_status() == "BL_OK"
    b = oracle.absmean_beta(W, eps)
    assert float(host(beta)[0]) == float(b)
    Xq, sc = oracle.act_quant(X, eps)
    for r0 in range(0, N, 4000):
        acc = oracle.contract(Xq, oracle.ternarize(W[r0:r0 + 4000], b))
        assert_y_exact(Y[:, r0:r0 + 4000], oracle.dequant(acc, sc, b))


def test_chain_output_feeds_next_input(bl):
    """Twelve GEMVs back to back on one stream, each reading the previous one's
    Y as its X (K = N), with static weights: the dependency wait must order
    every X read after the previous kernel's writes."""
    import torch
    K = N = 2560
    rng = np.random.default_rng(5)
    Ws = [(rng.standard_normal((N, K), dtype=np.float32) * F32(0.02 * (1 + i % 3))) for i in range(3)]
    Wq = [quantized(bl, _P(W)) for W in Ws]
    X0 = rng.standard_normal((1, K), dtype=np.float32)
    bufs = [dev(X0)] + [torch.empty((1, N), dtype=torch.float32, device="cuda") for _ in range(12)]
    for i in range(12):
        Wd, beta = Wq[i % 3]
        bl.linear(bufs[i], Wd, bl.PACK5, N, K, beta, out=bufs[i + 1], static_weights=True)
    assert bl.sync_status() == "BL_OK"
    x = X0
    for i in range(12):
        x = oracle.bitlinear(x, Ws[i % 3], 1e-5)["Y"]
        assert_y_exact(host(bufs[i + 1]), x)


def test_weights_rewritten_right_before_the_gemv(bl):
    """Without the static-weights flag the GEMV reads W only after the kernel
    before it has finished: quantize into the same packed buffer, then the
    linear, five times with different weights and no synchronization."""
    import torch
    K, N = 6912, 2560
    Wp = torch.empty((N, bl.pack5_ldp(K)), dtype=torch.uint8, device="cuda")
    beta = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = bl.workspace(bl.load().bl_quantize_weights_workspace_size(N, K), "cuda")
    outs, refs = [], []
    for i in range(5):
        p = random_problem(4000 + i, 1, K, N, w_sigma=0.01 * (i + 1))
        bl.quantize_weights_pack5(dev(p.W), p.eps, ws=ws, out=Wp, beta=beta)
        outs.append(bl.linear(dev(p.X), Wp, bl.PACK5, N, K, beta, eps=p.eps))
        refs.append(oracle.bitlinear(p.X, p.W, p.eps)["Y"])
    assert bl.sync_status() == "BL_OK"
    for Y, ref in zip(outs, refs):
        assert_y_exact(host(Y), ref)


def test_integer_product_with_static_weights(bl):
    """bl_linear_acc_ex on the GEMV with the flag: the exact integer product."""
    rng = np.random.default_rng(8)
    for M, K, N in ((1, 2560, 6912), (4, 6912, 2560), (3, 1001, 77)):
        Xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        Wq = rng.integers(-1, 2, (N, K)).astype(np.int8)
        acc = bl.linear_acc(dev(Xq), bl.pack(dev(Wq)), bl.PACK5, N, K, path=bl.PATH_GEMV, static_weights=True)
        assert bl.sync_status() == "BL_OK"
        np.testing.assert_array_equal(host(acc), oracle.contract(Xq, Wq))


def _pinned(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).pin_memory()


def test_group_host_buffers_back_to_back(bl):
    """bl_linear_group_host on the decode workload with both layers' rows back
    to back in one page-locked host buffer and one device buffer (each copy
    direction merged into one transfer): every output against the oracle, twice
    through the same marshalled call with new activations written in between."""
    import torch
    ps = list(problems(2))
    Ws = [quantized(bl, p) for p in ps]
    Kt = sum(p.K for p in ps)
    Nt = sum(p.N for p in ps)
    hx = torch.empty(Kt, dtype=torch.float32).pin_memory()
    hy = torch.full((Nt,), np.nan, dtype=torch.float32).pin_memory()
    dx = torch.empty(Kt, dtype=torch.float32, device="cuda")
    dy = torch.empty(Nt, dtype=torch.float32, device="cuda")
    calls, hX, hY, outs, k0, n0 = [], [], [], [], 0, 0
    for p, (Wd, beta) in zip(ps, Ws):
        calls.append((dx[k0:k0 + p.K].view(1, p.K), Wd, bl.PACK5, p.N, p.K, beta, None, p.eps))
        hX.append(hx[k0:k0 + p.K].view(1, p.K))
        hY.append(hy[n0:n0 + p.N].view(1, p.N))
        outs.append(dy[n0:n0 + p.N].view(1, p.N))
        k0, n0 = k0 + p.K, n0 + p.N
    g = bl.LinearGroupHost(calls, hX, hY, static_weights=True, outs=outs)
    for rep in range(2):
        Xs = [p.X if rep == 0 else np.random.default_rng(70 + i).standard_normal(p.X.shape).astype(F32) * 3
              for i, p in enumerate(ps)]
        for x, h in zip(Xs, hX):
            h.copy_(torch.from_numpy(x))
        g()
        torch.cuda.current_stream().synchronize()
        assert bl.sync_status() == "BL_OK"
        for x, p, h in zip(Xs, ps, hY):
            assert_y_exact(h.numpy(), oracle.bitlinear(x, p.W, p.eps)["Y"])


def test_group_host_buffers_mixed_calls(bl):
    """bl_linear_group_host over decode-GEMV, swapped tensor-core, unswapped
    tensor-core and one-trit-per-byte calls with separate host buffers: mapped
    page-locked rows read by the library's kernel (4-byte units, since one row
    block is not a whole number of 16-byte units), rows beyond the kernel's byte
    budget and a pageable pair moved by copies; decode results stored straight
    into host memory, the others copied back.  Every result equals the oracle's
    and bl_linear_group's."""
    import torch
    specs = [(1, 2560, 700), (1, 999, 1500), (2, 3000, 500), (64, 1040, 300), (3, 77, 90), (9, 640, 129),
             (300, 4000, 260), (1, 4096, 333)]
    calls, hX, hY, refs = [], [], [], []
    for i, (M, K, N) in enumerate(specs):
        p = random_problem(950 + i, M, K, N)
        fmt = bl.I8 if i == 4 else bl.PACK5
        Wd, beta = quantized(bl, p, fmt)
        bias = (np.random.default_rng(i).standard_normal(N) * 0.1).astype(F32) if i % 2 else None
        calls.append((torch.empty((M, K), dtype=torch.float32, device="cuda"), Wd, fmt, N, K, beta,
                      None if bias is None else dev(bias), p.eps))
        pageable = i == 1
        hX.append(torch.from_numpy(p.X.copy()) if pageable else _pinned(p.X))
        hY.append(torch.full((M, N), np.nan, dtype=torch.float32) if pageable
                  else torch.full((M, N), np.nan, dtype=torch.float32).pin_memory())
        refs.append(oracle.bitlinear(p.X, p.W, p.eps, bias)["Y"])
    assert sum(x.numel() * 4 for x in hX[:7]) > 4 << 20      # the last rows exceed the kernel's budget
    bl.linear_group_host(calls, hX, hY)
    torch.cuda.current_stream().synchronize()
    assert bl.sync_status() == "BL_OK"
    again = bl.linear_group(calls)
    for h, Y2, ref in zip(hY, again, refs):
        assert_y_exact(h.numpy(), ref)
        np.testing.assert_array_equal(host(Y2), h.numpy())


def test_group_host_buffers_with_an_empty_call(bl):
    """An M = 0 call inside a host-buffer group moves and computes nothing; the
    calls around it are exact (each host Y written, the empty one untouched)."""
    import torch
    specs = [(1, 2560, 300), (0, 640, 200), (2, 999, 129)]
    calls, hX, hY, refs = [], [], [], []
    for i, (M, K, N) in enumerate(specs):
        p = random_problem(990 + i, max(M, 1), K, N)
        Wd, beta = quantized(bl, p)
        X = p.X[:M]
        calls.append((torch.empty((M, K), dtype=torch.float32, device="cuda"), Wd, bl.PACK5, N, K, beta, None, p.eps))
        hX.append(_pinned(X))
        hY.append(torch.full((M, N), np.nan, dtype=torch.float32).pin_memory())
        refs.append(oracle.bitlinear(X, p.W, p.eps)["Y"] if M else None)
    bl.linear_group_host(calls, hX, hY, static_weights=True)
    torch.cuda.current_stream().synchronize()
    assert bl.sync_status() == "BL_OK"
    for h, ref in zip(hY, refs):
        if ref is not None:
            assert_y_exact(h.numpy(), ref)
        else:
            assert h.numel() == 0
