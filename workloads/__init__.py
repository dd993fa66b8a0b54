"""Seeded synthetic inputs for the BitLinear workloads.

This module only draws random numbers: it holds none of the layer's arithmetic
(no quantization, packing or contraction), so that the CPU oracle and the CUDA
path can both consume the same inputs without sharing any of the method.

The five workloads are the ones the BitLinear pages' layer is measured on:

1. ``tiny``         one BitLinear, W [256,128] ~ N(0, 0.02^2) stored one trit per
                    byte, X [8,128] ~ N(0,1), seed 0.
2. ``decode_gemv``  batch-1 decode: (K,N) = (2560,6912) and (6912,2560), packed
                    trits, W ~ N(0,0.02^2), X [1,K] ~ N(0,1) with floor(0.01 K)
                    distinct entries (drawn without replacement) scaled by 20, seed 1.
3. ``gpt_layers``   every BitLinear of a vocab-256, d_model-128, 4-layer, 4-head
                    ternary GPT: per layer Q,K,V,O 128->128, up 128->512,
                    down 512->128, tokens M = 8*256 = 2048, seed 2.  Each
                    matrix gets its own X ~ N(0,1) (not chained through a model).
4. ``prefill_gemm`` M = 4096: (K,N) = (4096,11008) and (11008,4096), packed, seed 3.
5. ``batch_sweep``  one K = N = 8192 layer, packed, W ~ U(-1,1)*0.05, X ~ N(0,1),
                    M in {1,2,4,8,16,32,64,128,256,1024}, seed 4.  W is drawn
                    once, then X [1024, 8192]; the case with M rows uses X[:M].

Draw recipe: ``numpy.random.default_rng(seed)`` (PCG64); normals are
``standard_normal(dtype=float32) * float32(sigma)``; uniforms are
``(random(dtype=float32) * 2 - 1) * float32(0.05)`` in float32; for each matrix
in order, W is drawn first, then X, then (workload 2) the outlier indices.
For data-parallel replicas, rank r > 0 seeds with ``[seed, r]`` so rank 0
always reproduces the single-GPU inputs.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Iterator, List, Optional, Tuple

import numpy as np

FMT_I8 = "i8"        # one trit per byte, [N, K] int8
FMT_PACK5 = "pack5"  # five trits per byte, [N, ldp] uint8

SWEEP_M = (1, 2, 4, 8, 16, 32, 64, 128, 256, 1024)


@dataclass(frozen=True)
class Workload:
    id: int
    name: str
    shapes: Tuple[Tuple[int, int, int], ...]   # (M, K, N) per BitLinear call
    fmt: str
    w_dist: Tuple                              # ("normal", sigma) | ("uniform", half_width)
    x_dist: Tuple                              # ("normal", 1.0) | ("normal_outliers", frac, scale)
    seed: int
    eps: float = 1e-5
    shared_weight: bool = False                # workload 5: one W, X rows sliced per M
    labels: Tuple[str, ...] = field(default=())


def _gpt_shapes():
    shapes, labels = [], []
    for layer in range(4):
        for name, (k, n) in (("q", (128, 128)), ("k", (128, 128)), ("v", (128, 128)),
                             ("o", (128, 128)), ("up", (128, 512)), ("down", (512, 128))):
            shapes.append((2048, k, n))
            labels.append(f"l{layer}.{name}")
    return tuple(shapes), tuple(labels)


_GPT_SHAPES, _GPT_LABELS = _gpt_shapes()

WORKLOADS = {
    1: Workload(1, "tiny", ((8, 128, 256),), FMT_I8, ("normal", 0.02), ("normal", 1.0), 0),
    2: Workload(2, "decode_gemv", ((1, 2560, 6912), (1, 6912, 2560)), FMT_PACK5,
                ("normal", 0.02), ("normal_outliers", 0.01, 20.0), 1),
    3: Workload(3, "gpt_layers", _GPT_SHAPES, FMT_I8, ("normal", 0.02), ("normal", 1.0), 2,
                labels=_GPT_LABELS),
    4: Workload(4, "prefill_gemm", ((4096, 4096, 11008), (4096, 11008, 4096)), FMT_PACK5,
                ("normal", 0.02), ("normal", 1.0), 3),
    5: Workload(5, "batch_sweep", tuple((m, 8192, 8192) for m in SWEEP_M), FMT_PACK5,
                ("uniform", 0.05), ("normal", 1.0), 4, shared_weight=True),
}


def rng_for(seed: int, rank: int = 0) -> np.random.Generator:
    return np.random.default_rng(seed if rank == 0 else [seed, rank])


def _draw_w(rng, dist, n, k):
    kind = dist[0]
    if kind == "normal":
        return rng.standard_normal((n, k), dtype=np.float32) * np.float32(dist[1])
    if kind == "uniform":
        u = rng.random((n, k), dtype=np.float32)
        return (u * np.float32(2) - np.float32(1)) * np.float32(dist[1])
    raise ValueError(kind)


def _draw_x(rng, dist, m, k):
    x = rng.standard_normal((m, k), dtype=np.float32)
    if dist[0] == "normal":
        return x * np.float32(dist[1]) if dist[1] != 1.0 else x
    if dist[0] == "normal_outliers":
        frac, scale = dist[1], dist[2]
        for r in range(m):
            idx = rng.choice(k, size=int(np.floor(frac * k)), replace=False)
            x[r, idx] *= np.float32(scale)
        return x
    raise ValueError(dist[0])


@dataclass
class Problem:
    """One BitLinear call's inputs: X [M,K] fp32 and W [N,K] fp32 (row-major)."""
    workload: int
    index: int
    label: str
    M: int
    K: int
    N: int
    X: np.ndarray
    W: np.ndarray
    fmt: str
    eps: float


def problems(wid: int, rank: int = 0, only: Optional[List[int]] = None) -> Iterator[Problem]:
    """Yield the workload's problems in draw order.

    ``only`` limits which problems are yielded; the draws of the skipped ones are
    still made so every problem's inputs are independent of the selection.
    """
    wl = WORKLOADS[wid]
    rng = rng_for(wl.seed, rank)
    if wl.shared_weight:
        mmax = max(s[0] for s in wl.shapes)
        _, k, n = wl.shapes[0]
        W = _draw_w(rng, wl.w_dist, n, k)
        X = _draw_x(rng, wl.x_dist, mmax, k)
        for i, (m, k2, n2) in enumerate(wl.shapes):
            if only is None or i in only:
                yield Problem(wid, i, f"M={m}", m, k, n, X[:m], W, wl.fmt, wl.eps)
        return
    for i, (m, k, n) in enumerate(wl.shapes):
        W = _draw_w(rng, wl.w_dist, n, k)
        X = _draw_x(rng, wl.x_dist, m, k)
        if only is None or i in only:
            label = wl.labels[i] if wl.labels else f"K={k},N={n}"
            yield Problem(wid, i, label, m, k, n, X, W, wl.fmt, wl.eps)


def random_problem(seed: int, M: int, K: int, N: int, w_sigma: float = 0.02,
                   x_sigma: float = 1.0, fmt: str = FMT_PACK5, eps: float = 1e-5) -> Problem:
    """A one-off Gaussian problem of any shape (parity cases, ragged tails)."""
    rng = np.random.default_rng(seed)
    W = _draw_w(rng, ("normal", w_sigma), N, K)
    X = _draw_x(rng, ("normal", x_sigma), M, K)
    return Problem(0, 0, f"M={M},K={K},N={N}", M, K, N, X, W, fmt, eps)
