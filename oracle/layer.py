"""Plain, slow, obviously correct BitLinear on the CPU (numpy).  Test infrastructure.

See the package docstring for the passages each function follows and the
readings taken where the pages are silent.
"""
from __future__ import annotations

import itertools
import math
from typing import Optional

import numpy as np

ACT_QMAX = 127          # symmetric int8 range [-127, 127] ("the bytes")
_F32 = np.float32


def absmean_beta(W: np.ndarray, eps: float) -> np.float32:
    """beta = (1/n) sum_i |W_i| + eps  ("the bytes", absmean equation).

    The sum is the exact real sum of the float32 magnitudes, rounded once to
    float64 (``math.fsum`` returns the correctly rounded sum); the mean is that
    float64 divided by n in float64, rounded to float32; eps is added in float32.
    """
    a = np.abs(np.asarray(W, dtype=_F32)).ravel()
    n = a.size
    if n == 0:
        raise ValueError("absmean of an empty tensor")
    if not np.all(np.isfinite(a)):
        raise ValueError("weights must be finite")
    step = 1 << 20
    chunks = (a[i:i + step].astype(np.float64).tolist() for i in range(0, n, step))
    total = math.fsum(itertools.chain.from_iterable(chunks))
    mean = total / n
    return _F32(_F32(mean) + _F32(eps))


def ternarize(W: np.ndarray, beta) -> np.ndarray:
    """W_q = clip(round(W / beta), -1, 1) in {-1, 0, +1}  ("the bytes").

    float32 division, round-half-to-even, then the clip; stored one trit per
    byte (int8), the pages' "1 edge = 1 byte" layout.
    """
    q = np.rint(np.asarray(W, dtype=_F32) / _F32(beta))
    return np.clip(q, -1, 1).astype(np.int8)


def pack5_ldp(K: int) -> int:
    """Packed row stride: ceil(K/5) bytes rounded up to a multiple of 16."""
    nb = -(-K // 5)
    return -(-nb // 16) * 16


def pack5(Wq: np.ndarray, ldp: Optional[int] = None) -> np.ndarray:
    """Five trits per byte: byte j of a row = sum_{k<5} (t_{5j+k} + 1) * 3^k.

    Trits beyond K are 0; bytes beyond ceil(K/5) up to ``ldp`` are therefore 121.
    """
    Wq = np.asarray(Wq)
    N, K = Wq.shape
    if ldp is None:
        ldp = pack5_ldp(K)
    if ldp * 5 < K:
        raise ValueError("ldp too small for K")
    trits = np.zeros((N, ldp * 5), dtype=np.int64)
    trits[:, :K] = Wq
    digits = (trits + 1).reshape(N, ldp, 5)
    out = np.zeros((N, ldp), dtype=np.int64)
    for k in range(5):
        out += digits[:, :, k] * (3 ** k)
    return out.astype(np.uint8)


def unpack5(Wp: np.ndarray, K: int) -> np.ndarray:
    """Inverse of ``pack5``: t_{5j+k} = floor(b_j / 3^k) mod 3 - 1, first K trits."""
    Wp = np.asarray(Wp).astype(np.int64)
    N, ldp = Wp.shape
    if np.any(Wp > 242):
        raise ValueError("packed byte above 3^5 - 1")
    trits = np.zeros((N, ldp, 5), dtype=np.int64)
    for k in range(5):
        trits[:, :, k] = (Wp // (3 ** k)) % 3 - 1
    return trits.reshape(N, ldp * 5)[:, :K].astype(np.int8)


def act_quant(X: np.ndarray, eps: float):
    """Per-row absmax int8 quantization ("the bytes"; per-token fix in "attention").

    s_m = max_k |X[m,k]| / 127 + eps (float32, division then addition);
    X_q = clip(round(X / s_m), -127, 127).  Returns (X_q int8 [M,K], s float32 [M]).
    """
    X = np.asarray(X, dtype=_F32)
    if X.ndim != 2:
        raise ValueError("X must be [M, K]")
    if not np.all(np.isfinite(X)):
        raise ValueError("activations must be finite")
    M, K = X.shape
    if K == 0:
        raise ValueError("K must be positive")
    amax = np.max(np.abs(X), axis=1) if M else np.zeros((0,), _F32)
    s = (amax / _F32(ACT_QMAX)) + _F32(eps)
    q = np.rint(X / s[:, None])
    return np.clip(q, -ACT_QMAX, ACT_QMAX).astype(np.int8), s.astype(_F32)


def contract(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc[m,n] = sum_k X_q[m,k] * W_q[n,k], exact in integers (x_q W_q^T)."""
    acc = np.asarray(Xq).astype(np.int64) @ np.asarray(Wq).astype(np.int64).T
    if acc.size and np.max(np.abs(acc)) >= 2 ** 31:
        raise OverflowError("accumulator exceeds int32")
    return acc.astype(np.int32)


def contract_f64(Xq: np.ndarray, Wq: np.ndarray) -> np.ndarray:
    """acc = x_q W_q^T as a float64 matrix product of the integer codes.

    The same definition as ``contract``, for full-size cases where an int64
    product is too slow: every product and every partial sum is an integer of
    magnitude at most 127 * K, far below 2^53, so float64 represents each one
    exactly and the result does not depend on how the library orders the sum.
    """
    Xq = np.asarray(Xq)
    Wq = np.asarray(Wq)
    if 127 * Xq.shape[1] >= 2 ** 53:
        raise OverflowError("partial sums may exceed 2^53")
    acc = Xq.astype(np.float64) @ Wq.astype(np.float64).T
    if acc.size and np.max(np.abs(acc)) >= 2 ** 31:
        raise OverflowError("accumulator exceeds int32")
    return acc.astype(np.int32)


def contract_entries(Xq_rows: np.ndarray, Wq_rows: np.ndarray) -> np.ndarray:
    """Selected outputs one by one: acc_i = sum_k Xq_rows[i,k] * Wq_rows[i,k]."""
    a = np.asarray(Xq_rows).astype(np.int64)
    b = np.asarray(Wq_rows).astype(np.int64)
    return np.einsum("ik,ik->i", a, b).astype(np.int32)


def dequant(acc: np.ndarray, s: np.ndarray, beta, bias: Optional[np.ndarray] = None):
    """y = float32(acc) * float32(s_m * beta) [+ b_n]  (deployed-path equation)."""
    acc = np.asarray(acc)
    if acc.size and np.max(np.abs(acc.astype(np.int64))) >= 2 ** 24:
        raise OverflowError("accumulator not exact in float32")
    sb = np.asarray(s, dtype=_F32) * _F32(beta)
    y = acc.astype(_F32) * sb.reshape(-1, *([1] * (acc.ndim - 1)))
    if bias is not None:
        y = y + np.asarray(bias, dtype=_F32)
    return y.astype(_F32)


def rmsnorm(X: np.ndarray, g: np.ndarray, eps_norm: float) -> np.ndarray:
    """RMSNorm(x) = x / sqrt((1/d) sum_i x_i^2 + eps) * g over the last dimension
    ("attention, as graph ops", RMSNorm equation; learnable gain g, float32).

    Reading, as for beta: the sum of squares is the exact real sum (each float32
    square is exact in float64), rounded once to float64 (``math.fsum``),
    divided by d in float64 and rounded to float32; then, all in float32:
    + eps, sqrt (correctly rounded), x / that, times g.
    """
    X = np.asarray(X, dtype=_F32)
    g = np.asarray(g, dtype=_F32)
    if X.ndim != 2 or g.shape != (X.shape[1],):
        raise ValueError("X must be [M, d] and g [d]")
    if not (np.all(np.isfinite(X)) and np.all(np.isfinite(g))):
        raise ValueError("inputs must be finite")
    M, d = X.shape
    out = np.empty_like(X)
    for m in range(M):
        S = math.fsum(float(v) * float(v) for v in X[m].tolist())
        ms = _F32(S / d)
        r = np.sqrt(_F32(ms + _F32(eps_norm)))
        out[m] = (X[m] / r) * g
    return out


def rmsnorm_act_quant(X: np.ndarray, g: np.ndarray, eps_norm: float, eps: float):
    """The pre-norm block's input to a BitLinear: x_q, s = act_quant(RMSNorm(x))
    (the PyPI page's block "x = x + mha(norm1(x))": the normalized rows are the
    layer's activations)."""
    return act_quant(rmsnorm(X, g, eps_norm), eps)


def bitlinear(X: np.ndarray, W: np.ndarray, eps: float = 1e-5,
              bias: Optional[np.ndarray] = None) -> dict:
    """The whole layer from float32 W and X: every intermediate is returned."""
    beta = absmean_beta(W, eps)
    Wq = ternarize(W, beta)
    Xq, s = act_quant(X, eps)
    acc = contract(Xq, Wq)
    Y = dequant(acc, s, beta, bias)
    return {"beta": beta, "Wq": Wq, "Xq": Xq, "s": s, "acc": acc, "Y": Y}
