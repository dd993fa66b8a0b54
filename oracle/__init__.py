"""CPU oracle for the BitLinear hot path.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its CPU-baseline
and reference legs) may import this package.  The product path never calls it:
the CUDA library has no CPU fallback.  The oracle shares no code with the CUDA
path; the two meet only in the seeded inputs of ``workloads``.

What it computes, and where the method is stated (page title, then section):

* ``absmean_beta`` and ``ternarize`` -- "ultragraph -- when the graph is the
  1-bit LLM, part 2", section "the bytes": beta = (1/n) sum_i |W_i| + eps,
  W_q = clip(round(W / beta), -1, 1).  One beta per weight tensor ("global beta"
  in section "autograd on a byte-graph, and the straight-through lie").
* ``act_quant`` -- same page, section "the bytes" and the per-token fix in
  section "attention, as graph ops": s = max_i |x_i| / 127 + eps per row,
  x_q = clip(round(x / s), -127, 127), the symmetric range [-127, 127].
* ``contract`` (and ``contract_f64``, the same product by a float64 matmul
  that is exact for these integer codes) and ``dequant`` -- same page, section
  "autograd on a byte-graph", deployed-path equation y = (x_q W_q^T)(s beta) + b: an integer matmul, then
  one rescale by the row scale times beta.
* ``pack5`` / ``unpack5`` -- "ultragraph-1bit 0.12.0" (PyPI), sections "A whole
  ternary GPT" and "Layout" (5 ternary values per byte, ~1.6 bits/weight), and
  "a 1-bit llm, from scratch", tl;dr (1.6 bits each).  Byte = sum_k (t_k+1) 3^k.

* ``rmsnorm`` and ``rmsnorm_act_quant`` -- part 2, section "attention, as graph
  ops" (RMSNorm equation, learnable gain g), and the PyPI page's pre-norm block
  "x = x + mha(norm1(x))": the normalized rows feed the BitLinear, so its
  activation quantization follows the norm.
* ``checkpoint.write_deployed`` / ``checkpoint.read_deployed`` -- "ultragraph-1bit
  0.12.0" (PyPI), section "A whole ternary GPT": the deployed checkpoint keeps
  the ternary weights at five per byte plus the float32 pieces (beta, biases),
  byte-exact; the file layout is read in ``oracle/checkpoint.py``.

* ``backward.ste_backward`` -- part 2, section "autograd on a byte-graph, and
  the straight-through lie": dL/dx = (dL/dy) W, dL/dW = (dL/dy)^T x,
  dL/db = sum of dL/dy, on the float32 masters, in float64.

Readings taken where the pages leave a step open:

1. Precision.  The pages' arrays are numpy float32, so every quantizer step is
   IEEE-754 float32 with round-to-nearest-even, in the order written.
2. The mean in beta is the exact real sum of |W| rounded once to float64
   (``math.fsum`` is correctly rounded), divided by n in float64, rounded to
   float32; eps is then added in float32.  A float32 running sum would make
   beta depend on summation order, which no two implementations share.
3. "round" is round-half-to-even (numpy's ``rint``/``round``).
4. eps is the same value in both quantizers (1e-5 unless a caller passes
   another) and is added after the mean / after max/127.
5. Dequantization multiplies s by beta first (the page's grouping "(s beta)"),
   then the float32 accumulator by that product, then adds b separately.
6. Packing runs along K in order: trit 5j+k of a row is digit k (little-endian)
   of byte j; trits past K are 0 (digit 1), so an all-padding byte is 121; the
   row stride ``ldp`` is ceil(K/5) rounded up to 16 bytes.

7. The deployed checkpoint's layout (the pages fix only its density and
   byte-exactness): little-endian records of name, N, K, flags, beta bits,
   the packed rows without their 16-byte padding, then the bias.

8. The straight-through backward uses the float32 master W and the float32
   input x (the page: the quantizers and the per-row scale are treated as the
   identity), not the dequantized beta W_q or s x_q.

9. RMSNorm's mean of squares is the exact sum of the float32 squares, rounded
   once to float64, divided by d in float64 and rounded to float32 (the reading
   of the mean in beta); + eps, sqrt, x / r and * g are float32 steps.  The
   norm's eps is its own argument, separate from the quantizers'.

Every function here is pinned (``tests/test_oracle_pins.py``,
``tests/test_oracle_checkpoint.py``, ``tests/test_oracle_backward.py``)
against hand-worked values, closed forms, invariants or brute force; none is
unpinned.
"""
from .layer import (  # noqa: F401
    ACT_QMAX,
    absmean_beta,
    act_quant,
    bitlinear,
    contract,
    contract_f64,
    contract_entries,
    dequant,
    pack5,
    pack5_ldp,
    rmsnorm,
    rmsnorm_act_quant,
    ternarize,
    unpack5,
)
