"""Plausible mistakes planted in the oracle (on the CPU) must fail a pin.

Each mutation is a wrong variant of one oracle step; the check is that at
least one of the pins in test_oracle_pins.py rejects it.  Nothing here runs on
the GPU.
"""
import math

import numpy as np
import pytest

import oracle
import oracle.layer as ob

F32 = np.float32


def _run_pins():
    return pytest.main(["-q", "-x", "-p", "no:cacheprovider",
                        __file__.replace("test_oracle_mutations.py", "test_oracle_pins.py")])


def _beta_f32_running_sum(W, eps):
    a = np.abs(np.asarray(W, F32)).ravel()
    tot = F32(0)
    for v in a:
        tot = F32(tot + v)
    return F32(F32(tot / F32(a.size)) + F32(eps))


def _ternarize_half_away(W, beta):
    q = np.trunc(np.asarray(W, F32) / F32(beta) + np.copysign(F32(0.5), W))
    return np.clip(q, -1, 1).astype(np.int8)


def _act_quant_half_away(X, eps):
    X = np.asarray(X, F32)
    s = np.max(np.abs(X), axis=1) / F32(127) + F32(eps)
    r = X / s[:, None]
    q = np.trunc(r + np.copysign(F32(0.5), r))
    return np.clip(q, -127, 127).astype(np.int8), s.astype(F32)


def _act_quant_per_tensor(X, eps):
    X = np.asarray(X, F32)
    s = np.full(X.shape[0], np.max(np.abs(X)) / F32(127) + F32(eps), F32)
    return np.clip(np.rint(X / s[:, None]), -127, 127).astype(np.int8), s


def _act_quant_128(X, eps):
    X = np.asarray(X, F32)
    s = np.max(np.abs(X), axis=1) / F32(128) + F32(eps)
    return np.clip(np.rint(X / s[:, None]), -128, 127).astype(np.int8), s.astype(F32)


def _pack_big_endian(Wq, ldp=None):
    Wq = np.asarray(Wq)
    N, K = Wq.shape
    ldp = ldp or ob.pack5_ldp(K)
    t = np.zeros((N, ldp * 5), np.int64)
    t[:, :K] = Wq
    d = (t + 1).reshape(N, ldp, 5)
    return sum(d[:, :, k] * 3 ** (4 - k) for k in range(5)).astype(np.uint8)


def _contract_transposed_w(Xq, Wq):
    Wq = np.asarray(Wq)
    if Wq.shape[0] == Wq.shape[1]:
        Wq = Wq.T
    return (np.asarray(Xq).astype(np.int64) @ Wq.astype(np.int64).T).astype(np.int32)


def _contract_f64_no_widening(Xq, Wq):
    return (np.asarray(Xq) @ np.asarray(Wq).T).astype(np.int32)   # int8 sums wrap


def _write_deployed_padded_rows(layers):
    import struct
    from oracle import checkpoint as ck
    out = [ck.MAGIC, struct.pack("<III", ck.VERSION, len(layers), 0)]
    for L in layers:
        name = L.get("name", "").encode()
        Wq = np.asarray(L["Wq"])
        N, K = Wq.shape
        bias = L.get("bias")
        out += [struct.pack("<I", len(name)), name,
                struct.pack("<QQII", N, K, 1 if bias is not None else 0,
                            int(np.float32(L["beta"]).view(np.uint32))),
                ob.pack5(Wq).tobytes()]                       # rows keep their 16-byte padding
        if bias is not None:
            out.append(np.asarray(bias, "<f4").tobytes())
    return b"".join(out)


def _dequant_acc_times_s_first(acc, s, beta, bias=None):
    y = (np.asarray(acc).astype(F32) * np.asarray(s, F32).reshape(-1, 1)) * F32(beta)
    return y if bias is None else y + np.asarray(bias, F32)


def _beta_no_eps(W, eps):
    return ob.absmean_beta(W, 0.0)


MUTANTS = {
    "absmean_beta": [_beta_f32_running_sum, _beta_no_eps],
    "ternarize": [_ternarize_half_away],
    "act_quant": [_act_quant_half_away, _act_quant_per_tensor, _act_quant_128],
    "pack5": [_pack_big_endian],
    "contract": [_contract_transposed_w],
    "contract_f64": [_contract_f64_no_widening],
    "dequant": [_dequant_acc_times_s_first],
}


def _ste_dequantized(dY, X, W):
    from oracle import backward as bw
    import oracle as o
    beta = o.absmean_beta(W, 1e-5)
    Wd = o.ternarize(W, beta).astype(np.float32) * np.float32(beta)
    return bw.__dict__["_orig"](dY, X, Wd)


def _ste_transposed(dY, X, W):
    dY, X, W = (np.asarray(a, np.float64) for a in (dY, X, W))
    return dY @ W, X.T @ dY if X.shape[1] == dY.shape[1] else (dY.T @ X), dY.sum(0)


def _ste_db_mean(dY, X, W):
    dX, dW, db = __import__("oracle.backward", fromlist=["x"]).__dict__["_orig"](dY, X, W)
    return dX, dW, db / np.asarray(dY).shape[0]


@pytest.mark.parametrize("mutant", [_ste_dequantized, _ste_transposed, _ste_db_mean],
                         ids=lambda f: f.__name__)
def test_backward_pins_reject_mutant(mutant, monkeypatch):
    from oracle import backward as bw
    monkeypatch.setattr(bw, "_orig", bw.ste_backward, raising=False)
    monkeypatch.setattr(bw, "ste_backward", mutant)
    rc = pytest.main(["-q", "-x", "-p", "no:cacheprovider",
                      __file__.replace("test_oracle_mutations.py", "test_oracle_backward.py")])
    assert rc != 0


def _rms_sum_not_mean(X, g, eps):
    X = np.asarray(X, F32)
    out = np.empty_like(X)
    for m in range(X.shape[0]):
        S = math.fsum(float(v) * float(v) for v in X[m])
        out[m] = (X[m] / np.sqrt(F32(F32(S) + F32(eps)))) * np.asarray(g, F32)
    return out


def _rms_float32_running_sum(X, g, eps):
    X = np.asarray(X, F32)
    out = np.empty_like(X)
    for m in range(X.shape[0]):
        S = F32(0)
        for v in X[m]:
            S = F32(S + F32(v * v))
        out[m] = (X[m] / np.sqrt(F32(F32(S / F32(X.shape[1])) + F32(eps)))) * np.asarray(g, F32)
    return out


def _rms_eps_outside_sqrt(X, g, eps):
    X = np.asarray(X, F32)
    out = np.empty_like(X)
    for m in range(X.shape[0]):
        S = math.fsum(float(v) * float(v) for v in X[m])
        out[m] = (X[m] / F32(np.sqrt(F32(S / X.shape[1])) + F32(eps))) * np.asarray(g, F32)
    return out


@pytest.mark.parametrize("mutant", [_rms_sum_not_mean, _rms_float32_running_sum, _rms_eps_outside_sqrt],
                         ids=lambda f: f.__name__)
def test_rmsnorm_pins_reject_mutant(mutant, monkeypatch):
    monkeypatch.setattr(ob, "rmsnorm", mutant)
    monkeypatch.setattr(oracle, "rmsnorm", mutant)
    rc = pytest.main(["-q", "-x", "-p", "no:cacheprovider",
                      __file__.replace("test_oracle_mutations.py", "test_oracle_rmsnorm.py")])
    assert rc != 0


def test_checkpoint_pins_reject_padded_rows(monkeypatch):
    from oracle import checkpoint as ck
    monkeypatch.setattr(ck, "write_deployed", _write_deployed_padded_rows)
    rc = pytest.main(["-q", "-x", "-p", "no:cacheprovider",
                      __file__.replace("test_oracle_mutations.py", "test_oracle_checkpoint.py")])
    assert rc != 0


@pytest.mark.parametrize("name,mutant", [(n, f) for n, fs in MUTANTS.items() for f in fs],
                         ids=lambda v: getattr(v, "__name__", v))
def test_pins_reject_mutant(name, mutant, monkeypatch):
    monkeypatch.setattr(ob, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    assert _run_pins() != 0, f"pins did not catch {mutant.__name__}"
