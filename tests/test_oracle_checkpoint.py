"""Pins of the deployed-checkpoint oracle (oracle/checkpoint.py): hand-worked
bytes, the round trip, the record sizes and the 1.6-bit density the pages
state ("ultragraph-1bit 0.12.0" (PyPI), section "A whole ternary GPT")."""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import checkpoint

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "deployed_hand.json")))


def _layers_from_gold():
    out = []
    for L in GOLD["layers"]:
        d = {"name": L["name"], "Wq": np.array(L["Wq"], np.int8), "beta": np.float32(L["beta"])}
        if L["bias"] is not None:
            d["bias"] = np.array(L["bias"], np.float32)
        out.append(d)
    return out


def test_hand_worked_bytes():
    data = checkpoint.write_deployed(_layers_from_gold())
    assert data.hex().upper() == GOLD["bytes_hex"].upper()
    back = checkpoint.read_deployed(bytes.fromhex(GOLD["bytes_hex"]))
    assert [b["name"] for b in back] == ["l0", ""]
    np.testing.assert_array_equal(back[0]["packed"], [[146, 123], [121, 121]])
    np.testing.assert_array_equal(back[0]["Wq"], GOLD["layers"][0]["Wq"])
    assert back[0]["bias"] is None and back[1]["bias"].tolist() == [2.0]
    assert back[0]["beta"] == np.float32(0.25) and back[1]["beta"] == np.float32(1.5)


@pytest.mark.parametrize("K", [5, 6, 7, 8, 9, 2560, 6913])
def test_round_trip_and_sizes(K):
    rng = np.random.default_rng(K)
    layers = []
    for i, N in enumerate((1, 3, 17)):
        d = {"name": f"blocks.{i}.ff", "Wq": rng.integers(-1, 2, (N, K)).astype(np.int8),
             "beta": np.float32(rng.random() * 0.1)}
        if i % 2:
            d["bias"] = rng.standard_normal(N).astype(np.float32)
        layers.append(d)
    data = checkpoint.write_deployed(layers)
    size = 16 + sum(4 + len(d["name"]) + 24 + d["Wq"].shape[0] * -(-K // 5) +
                    (4 * d["Wq"].shape[0] if "bias" in d else 0) for d in layers)
    assert len(data) == size
    back = checkpoint.read_deployed(data)
    for d, b in zip(layers, back):
        assert b["name"] == d["name"] and (b["N"], b["K"]) == d["Wq"].shape
        np.testing.assert_array_equal(b["Wq"], d["Wq"])
        np.testing.assert_array_equal(b["packed"], oracle.pack5(d["Wq"])[:, :-(-K // 5)])
        assert b["beta"].view(np.uint32) == np.float32(d["beta"]).view(np.uint32)
        if "bias" in d:
            np.testing.assert_array_equal(b["bias"], d["bias"])
        else:
            assert b["bias"] is None
    assert checkpoint.write_deployed(back) == data          # byte-exact both ways


def test_density_is_1_6_bits_per_weight():
    """Five trits per byte: the weights of a K = 5j layer take 8/5 bits each."""
    N, K = 64, 640
    Wq = np.zeros((N, K), np.int8)
    data = checkpoint.write_deployed([{"name": "", "Wq": Wq, "beta": np.float32(1)}])
    weight_bytes = len(data) - 16 - 4 - 24
    assert weight_bytes * 8 / (N * K) == pytest.approx(1.6)


def test_rejects_malformed_files():
    good = bytes.fromhex(GOLD["bytes_hex"])
    for bad in (b"", b"XXXX" + good[4:], good[:-1], good + b"\0",
                good[:4] + (2).to_bytes(4, "little") + good[8:]):
        with pytest.raises(ValueError):
            checkpoint.read_deployed(bad)
