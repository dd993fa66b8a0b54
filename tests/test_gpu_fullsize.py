"""Full-size workloads checked against the oracle element by element.

The prefill shapes (M = 4096, (K, N) = (4096, 11008) and (11008, 4096)) and the
batch sweep (K = N = 8192, M = 1 .. 1024) run on the tensor cores with more
output tiles than SMs, so every persistent CTA walks several work items and
both TMEM accumulators.  Every element of Y and of the int32 accumulators is
compared with the oracle: beta, codes and row scales from ``oracle``, the
exact integer product from ``oracle.contract_f64`` (pinned against
``oracle.contract``), then ``oracle.dequant``.  Three routes are covered:
bl_linear (activation quantization, packed weights unpacked once, GEMM),
bl_linear_acc with no workspace (trits decoded inside the GEMM at any M) and
bl_linear_acc_ex with a workspace (the unpack route for the integer product).
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
    bad = np.argwhere(y != ref)
    assert bad.size == 0, f"{len(bad)} outputs differ, first at {bad[:4].tolist()}"


def assert_acc_exact(acc, ref):
    bad = np.argwhere(acc != ref)
    assert bad.size == 0, f"{len(bad)} accumulators differ, first at {bad[:4].tolist()}"


def reference(p, beta=None):
    """Every intermediate of the layer from the oracle, at full size."""
    rb = oracle.absmean_beta(p.W, p.eps) if beta is None else beta
    Wq = oracle.ternarize(p.W, rb)
    Xq, s = oracle.act_quant(p.X, p.eps)
    acc = oracle.contract_f64(Xq, Wq)
    return {"beta": rb, "Wq": Wq, "Xq": Xq, "s": s, "acc": acc, "Y": oracle.dequant(acc, s, rb)}


def run_routes(bl, p, Wd, beta_d):
    """Y through bl_linear, acc through both bl_linear_acc routes."""
    import torch
    Xd = dev(p.X)
    Y = host(bl.linear(Xd, Wd, bl.PACK5, p.N, p.K, beta_d, eps=p.eps))
    Xq_d, s_d = bl.quantize_act(Xd, p.eps)
    acc_dec = torch.empty((p.M, p.N), dtype=torch.int32, device="cuda")
    lib = bl.load()
    code = lib.bl_linear_acc(Xq_d.data_ptr(), p.M, p.K, Wd.data_ptr(), bl.PACK5, p.N, Wd.shape[1],
                             acc_dec.data_ptr(), None)
    assert bl.STATUS[code] == "BL_OK"
    acc_unp = bl.linear_acc(Xq_d, Wd, bl.PACK5, p.N, p.K, path=bl.PATH_TC)
    assert bl.sync_status() == "BL_OK"
    return Y, host(Xq_d), host(s_d), host(acc_dec), host(acc_unp)


@pytest.mark.parametrize("idx", [0, 1])
def test_prefill_every_element(bl, idx):
    p = next(problems(4, only=[idx]))
    Wd, beta_d = bl.quantize_weights_pack5(dev(p.W), p.eps)
    ref = reference(p)
    assert host(beta_d)[0] == ref["beta"]
    np.testing.assert_array_equal(host(Wd), oracle.pack5(ref["Wq"]))
    path, _ = bl.linear_plan(p.M, p.N, p.K, bl.PACK5)
    assert path == bl.PATH_TC
    Y, Xq, s, acc_dec, acc_unp = run_routes(bl, p, Wd, beta_d)
    np.testing.assert_array_equal(s, ref["s"])
    np.testing.assert_array_equal(Xq, ref["Xq"])
    assert_acc_exact(acc_dec, ref["acc"])
    assert_acc_exact(acc_unp, ref["acc"])
    assert_y_exact(Y, ref["Y"])


def test_batch_sweep_every_element(bl):
    """One W, X[:M] for every M of the sweep; rows are independent (per-token
    scales), so the oracle's 1024-row result gives every case's first M rows."""
    ps = list(problems(5))
    p_all = ps[-1]
    assert p_all.M == 1024
    Wd, beta_d = bl.quantize_weights_pack5(dev(p_all.W), p_all.eps)
    ref = reference(p_all)
    assert host(beta_d)[0] == ref["beta"]
    np.testing.assert_array_equal(host(Wd), oracle.pack5(ref["Wq"]))
    for p in ps:
        Y, Xq, s, acc_dec, acc_unp = run_routes(bl, p, Wd, beta_d)
        m = p.M
        np.testing.assert_array_equal(Xq, ref["Xq"][:m])
        assert_acc_exact(acc_dec, ref["acc"][:m])
        assert_acc_exact(acc_unp, ref["acc"][:m])
        assert_y_exact(Y, ref["Y"][:m])


@pytest.mark.parametrize("fmt", ["i8", "pack5"])
@pytest.mark.parametrize("M,K,N", [(768, 256, 6400), (1024, 384, 9472), (700, 1040, 8000)])
def test_more_tiles_than_sms(bl, fmt, M, K, N):
    """150 to 296 output tiles of 128 x 256 on 148 SMs at modest K, both weight
    formats (packed: the unpack route, M > 512); ragged M, N and K tails."""
    f = bl.PACK5 if fmt == "pack5" else bl.I8
    p = random_problem(M + K + N + (f == bl.PACK5), M, K, N)
    assert -(-M // 128) * -(-N // 256) > 148
    assert bl.linear_plan(M, N, K, f)[0] == bl.PATH_TC
    Wfn = bl.quantize_weights_pack5 if f == bl.PACK5 else bl.quantize_weights
    Wd, beta_d = Wfn(dev(p.W), p.eps)
    bias = np.random.default_rng(M).standard_normal(N).astype(F32)
    Y = host(bl.linear(dev(p.X), Wd, f, N, K, beta_d, dev(bias), eps=p.eps))
    Xq_d, _ = bl.quantize_act(dev(p.X), p.eps)
    acc = host(bl.linear_acc(Xq_d, Wd, f, N, K, path=bl.PATH_TC))
    assert bl.sync_status() == "BL_OK"
    rb = oracle.absmean_beta(p.W, p.eps)
    assert host(beta_d)[0] == rb
    Wq = oracle.ternarize(p.W, rb)
    Xq, s = oracle.act_quant(p.X, p.eps)
    ref_acc = oracle.contract_f64(Xq, Wq)
    assert_acc_exact(acc, ref_acc)
    assert_y_exact(Y, oracle.dequant(ref_acc, s, rb, bias))
