"""Deployed checkpoint of BitLinear layers, written and read in plain Python.
Test infrastructure only (see the package docstring).

"ultragraph-1bit 0.12.0" (PyPI), section "A whole ternary GPT": the deployed
checkpoint keeps the ternary weights at their packed density, five trits per
byte, plus the small float32 pieces, and a model loaded from it computes the
same outputs as the one that wrote it, straight from the stored bytes.  The
pages fix the density and the byte-exactness, not a file layout; this is the
plainest layout that carries a BitLinear layer (reading recorded with the
others): little-endian throughout, no alignment padding.

    file   := header layer*
    header := b"BLT5"  version:u32 = 1  count:u32  reserved:u32 = 0
    layer  := name_len:u32 (<= 255)  name:name_len bytes (UTF-8)
              N:u64  K:u64  flags:u32 (bit 0: a bias follows)  beta:u32 (float32 bits)
              packed:N * ceil(K/5) bytes  (row n, byte j = sum_k (t_{5j+k}+1) 3^k, trits past K = 0)
              [bias:N float32]

The packed rows are exactly ``pack5`` of the codes without the row padding,
so the weights take 8/5 = 1.6 bits each when 5 divides K.
"""
from __future__ import annotations

import struct
from typing import List, Optional

import numpy as np

from .layer import pack5, unpack5

MAGIC = b"BLT5"
VERSION = 1


def write_deployed(layers: List[dict]) -> bytes:
    """layers: dicts with name (str), Wq (int8 [N, K] codes), beta (float32) and
    optionally bias (float32 [N]).  Returns the file's bytes."""
    out = [MAGIC, struct.pack("<III", VERSION, len(layers), 0)]
    for L in layers:
        name = L.get("name", "").encode("utf-8")
        if len(name) > 255:
            raise ValueError("layer name longer than 255 bytes")
        Wq = np.asarray(L["Wq"])
        N, K = Wq.shape
        cb = -(-K // 5)
        packed = pack5(Wq)[:, :cb]
        bias: Optional[np.ndarray] = L.get("bias")
        beta_bits = np.float32(L["beta"]).view(np.uint32)
        out.append(struct.pack("<I", len(name)))
        out.append(name)
        out.append(struct.pack("<QQII", N, K, 1 if bias is not None else 0, int(beta_bits)))
        out.append(np.ascontiguousarray(packed, dtype=np.uint8).tobytes())
        if bias is not None:
            b = np.asarray(bias, dtype=np.float32)
            if b.shape != (N,):
                raise ValueError("bias must be [N]")
            out.append(b.astype("<f4").tobytes())
    return b"".join(out)


def read_deployed(data: bytes) -> List[dict]:
    """The layers of a deployed checkpoint: name, N, K, beta, packed
    [N, ceil(K/5)], Wq (the unpacked codes) and bias (or None)."""
    if len(data) < 16 or data[:4] != MAGIC:
        raise ValueError("not a deployed BitLinear checkpoint")
    version, count, _ = struct.unpack_from("<III", data, 4)
    if version != VERSION:
        raise ValueError("unknown checkpoint version")
    off, layers = 16, []
    for _ in range(count):
        (nlen,) = struct.unpack_from("<I", data, off)
        off += 4
        if nlen > 255:
            raise ValueError("layer name longer than 255 bytes")
        name = data[off:off + nlen].decode("utf-8")
        off += nlen
        N, K, flags, beta_bits = struct.unpack_from("<QQII", data, off)
        off += 24
        cb = -(-K // 5)
        nb = N * cb
        if off + nb > len(data):
            raise ValueError("truncated checkpoint")
        packed = np.frombuffer(data, dtype=np.uint8, count=nb, offset=off).reshape(N, cb).copy()
        off += nb
        bias = None
        if flags & 1:
            if off + 4 * N > len(data):
                raise ValueError("truncated checkpoint")
            bias = np.frombuffer(data, dtype="<f4", count=N, offset=off).astype(np.float32)
            off += 4 * N
        layers.append({"name": name, "N": N, "K": K,
                       "beta": np.uint32(beta_bits).view(np.float32),
                       "packed": packed, "Wq": unpack5(packed, K), "bias": bias})
    if off != len(data):
        raise ValueError("trailing bytes after the last layer")
    return layers
