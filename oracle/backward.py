"""Straight-through backward of the BitLinear layer, in plain numpy float64.
Test infrastructure only (see the package docstring).

"ultragraph -- when the graph is the 1-bit LLM, part 2", section "autograd on a
byte-graph, and the straight-through lie": the forward runs on the quantized
bytes, y = (x_q W_q^T)(s beta) + b, but the backward treats the quantizers
and the per-row scale as the identity and routes the gradient into the
full-precision masters:

    dL/dx = (dL/dy) W,     dL/dW = (dL/dy)^T x,     dL/db = sum over rows of dL/dy

with W the float32 master weights [N, K], x the float32 layer input [M, K]
and dL/dy [M, N].  The same section's matmul rule (for C = A B, dL/dA =
dL/dC B^T and dL/dB = A^T dL/dC) is what these three lines instantiate.

The products here are float64 matmuls of the float32 inputs (each product is
exact in float64; the sums carry float64 rounding, far below float32's), so
they stand in for the exact real results against which a float32 kernel is
judged.  ``abs_bound`` gives the matching sums of |products|, the scale of the
componentwise error bound of a float32 GEMM.
"""
from __future__ import annotations

import numpy as np


def ste_backward(dY: np.ndarray, X: np.ndarray, W: np.ndarray):
    """(dX [M,K], dW [N,K], db [N]) in float64 from float32 dY [M,N], X [M,K], W [N,K]."""
    dY = np.asarray(dY, np.float32).astype(np.float64)
    X = np.asarray(X, np.float32).astype(np.float64)
    W = np.asarray(W, np.float32).astype(np.float64)
    if dY.shape[0] != X.shape[0] or dY.shape[1] != W.shape[0] or X.shape[1] != W.shape[1]:
        raise ValueError("shapes must be dY [M,N], X [M,K], W [N,K]")
    dX = dY @ W
    dW = dY.T @ X
    db = dY.sum(axis=0)
    return dX, dW, db


def abs_bound(dY: np.ndarray, X: np.ndarray, W: np.ndarray):
    """Sums of |products| behind each output: |dY| |W|, |dY|^T |X|, sum |dY|."""
    a = np.abs(np.asarray(dY, np.float32).astype(np.float64))
    return (a @ np.abs(np.asarray(W, np.float64)), a.T @ np.abs(np.asarray(X, np.float64)), a.sum(axis=0))
