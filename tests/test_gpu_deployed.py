"""The deployed checkpoint through the C ABI against the oracle's writer and
reader ("ultragraph-1bit 0.12.0" (PyPI), section "A whole ternary GPT"): the
library writes the oracle's bytes from device buffers, reads the oracle's
files into device buffers bit for bit, and a layer loaded from the file
computes exactly the outputs of the layer that wrote it."""
import numpy as np
import pytest

import oracle
from oracle import checkpoint
from workloads import random_problem

pytestmark = pytest.mark.gpu
F32 = np.float32


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.cpu().numpy()


SHAPES = [("blocks.0.attn.q", 1, 128, 128), ("blocks.0.ff.up", 1, 2560, 700), ("lm", 3, 333, 70),
          ("odd", 2, 6913, 9)]


def _device_layers(bl):
    out = []
    for i, (name, M, K, N) in enumerate(SHAPES):
        p = random_problem(300 + i, M, K, N)
        Wp, beta = bl.quantize_weights_pack5(dev(p.W), p.eps)
        bias = (np.random.default_rng(i).standard_normal(N) * 0.1).astype(F32) if i % 2 else None
        out.append({"name": name, "p": p, "Wp": Wp, "K": K, "beta": beta,
                    "bias": None if bias is None else dev(bias), "bias_h": bias})
    return out


def _oracle_layers(layers):
    res = []
    for L in layers:
        rb = oracle.absmean_beta(L["p"].W, L["p"].eps)
        d = {"name": L["name"], "Wq": oracle.ternarize(L["p"].W, rb), "beta": rb}
        if L["bias_h"] is not None:
            d["bias"] = L["bias_h"]
        res.append(d)
    return res


def test_save_writes_the_oracle_bytes(bl, tmp_path):
    layers = _device_layers(bl)
    path = str(tmp_path / "model.blt")
    bl.save_deployed(path, layers)
    assert bl.sync_status() == "BL_OK"
    with open(path, "rb") as fh:
        data = fh.read()
    assert data == checkpoint.write_deployed(_oracle_layers(layers))


def test_load_reads_the_oracle_file_and_runs_from_it(bl, tmp_path):
    layers = _device_layers(bl)
    ref = _oracle_layers(layers)
    path = tmp_path / "oracle.blt"
    path.write_bytes(checkpoint.write_deployed(ref))
    loaded = bl.load_deployed(str(path))
    assert bl.sync_status() == "BL_OK"
    assert [L["name"] for L in loaded] == [L["name"] for L in layers]
    for L, R, orig in zip(loaded, ref, layers):
        np.testing.assert_array_equal(host(L["Wp"]), oracle.pack5(R["Wq"]))      # 121 in the row padding
        assert host(L["beta"]).view(np.uint32)[0] == np.float32(R["beta"]).view(np.uint32)
        if "bias" in R:
            np.testing.assert_array_equal(host(L["bias"]), R["bias"])
        else:
            assert L["bias"] is None
        p = orig["p"]
        Y = host(bl.linear(dev(p.X), L["Wp"], bl.PACK5, p.N, p.K, L["beta"], L["bias"], p.eps))
        Y0 = host(bl.linear(dev(p.X), orig["Wp"], bl.PACK5, p.N, p.K, orig["beta"], orig["bias"], p.eps))
        np.testing.assert_array_equal(Y, Y0)
        np.testing.assert_array_equal(Y, oracle.bitlinear(p.X, p.W, p.eps, R.get("bias"))["Y"])
    # save what was loaded: the same bytes again
    again = str(tmp_path / "again.blt")
    bl.save_deployed(again, [{"name": L["name"], "Wp": L["Wp"], "K": L["K"], "beta": L["beta"], "bias": L["bias"]}
                             for L in loaded])
    with open(again, "rb") as fh:
        assert fh.read() == path.read_bytes()


def test_load_rejects_a_byte_that_is_not_a_code(bl, tmp_path):
    import ctypes
    import torch
    data = bytearray(checkpoint.write_deployed([{"name": "x", "Wq": np.zeros((3, 10), np.int8),
                                                 "beta": np.float32(1)}]))
    data[-1] = 243
    path = tmp_path / "bad.blt"
    path.write_bytes(bytes(data))
    Wp = torch.zeros((3, 16), dtype=torch.uint8, device="cuda")
    beta = torch.zeros(1, dtype=torch.float32, device="cuda")
    code = bl.load().bl_load_deployed_layer(str(path).encode(), 0, Wp.data_ptr(), 16, beta.data_ptr(), None,
                                            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert bl.STATUS[code] == "BL_ERR_IO"
