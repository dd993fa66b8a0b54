/*
 * bitlinear.h -- C ABI of a B200 (sm_100a) BitLinear library: ternary weights
 * times per-row absmax int8 activations, accumulated exactly in int32.
 *
 * The operation follows "ultragraph -- when the graph is the 1-bit LLM, part 2":
 *   section "the bytes":
 *     beta = (1/n) sum_i |W_i| + eps,   W_q = clip(round(W / beta), -1, 1)
 *     s    = max_i |x_i| / 127 + eps,   x_q = clip(round(x / s), -127, 127)
 *   section "autograd on a byte-graph, and the straight-through lie":
 *     y = (x_q W_q^T)(s beta) + b        (the deployed forward path)
 * and the dense trit format of "ultragraph-1bit 0.12.0" (PyPI), sections
 * "A whole ternary GPT" and "Layout": five ternary values per byte.
 *
 * Conventions shared by every entry point
 *   - Matrices are row-major.  W is [N, K] (out x in), X is [M, K], Y is [M, N].
 *   - Every pointer argument is a DEVICE pointer owned by the caller (except the
 *     host buffers of bl_linear_group_host and the checkpoint paths); the library
 *     allocates no device memory.  Scratch memory is passed in as `ws` (device, 256-byte
 *     aligned) with a size from the matching *_workspace_size function.
 *   - Calls are asynchronous on `stream` (NULL = the legacy default stream).  A
 *     validation error returns at once and launches nothing.  A failed launch
 *     returns BL_ERR_CUDA.  Conditions found on the device (non-finite inputs,
 *     a bounded wait that gave up) are recorded in a per-device status word and
 *     reported by bl_sync_status().
 *   - Arithmetic is IEEE-754 float32, round-to-nearest-even, in the order the
 *     formulas are written; no step is contracted into an FMA.  "round" is
 *     round-half-to-even.  Trit codes, int8 codes, scales, beta and int32
 *     accumulators are exact; Y is the float32 product acc * (s * beta) [+ b].
 *   - The mean in beta is the exact real sum of |W|, rounded once to float64,
 *     divided by n in float64, rounded to float32; eps is added in float32.
 *   - Inputs must be finite; eps must be finite and > 0; 1 <= K <= 131072 so
 *     that every accumulator (|acc| <= 127 K < 2^24) is exact in float32.
 *   - No C++ exception crosses this boundary.
 */
#ifndef BITLINEAR_H_
#define BITLINEAR_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h> /* cudaStream_t */

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  BL_OK = 0,
  BL_ERR_INVALID_ARG = 1,    /* null pointer, bad size, eps <= 0, K out of range */
  BL_ERR_ALIGNMENT = 2,      /* a pointer or stride breaks the stated alignment */
  BL_ERR_UNSUPPORTED = 3,    /* a forced kernel path cannot take this shape */
  BL_ERR_WORKSPACE = 4,      /* ws NULL, too small, unaligned, or (device) not cleared */
  BL_ERR_CUDA = 5,           /* a CUDA runtime call or launch failed */
  BL_ERR_DEVICE_TIMEOUT = 6, /* a bounded device-side wait gave up */
  BL_ERR_NONFINITE = 7,      /* a kernel met a NaN or Inf input */
  BL_ERR_IO = 8              /* a checkpoint file could not be written or read, or is malformed */
} bl_status;

/* Weight storage formats. */
typedef enum {
  /* One trit per byte, int8 in {-1,0,+1}, [N, ldw] with ldw >= K: the pages'
   * "1 edge = 1 byte" layout ("the bytes"). */
  BL_W_I8 = 0,
  /* Five trits per byte, uint8 [N, ldw], ldw = bl_pack5_ldp(K) or any larger
   * multiple of 16.  Byte j of row n is sum_{k<5} (W_q[n,5j+k] + 1) * 3^k, trits
   * past K count as 0, so whole padding bytes are 121 ("A whole ternary GPT"). */
  BL_W_PACK5 = 1
} bl_wfmt;

/* Kernel selection for the *_ex entry points (tests and benchmarks pin a path). */
typedef enum {
  BL_PATH_AUTO = 0, /* dispatch on M, K, N and the format */
  BL_PATH_SIMT = 1, /* dp4a tile kernel: any shape, any format */
  BL_PATH_GEMV = 2, /* packed-trit decode GEMV on CUDA cores: BL_W_PACK5, M <= 4; one
                       launch, activation quantization inside */
  BL_PATH_TC = 3    /* tcgen05 kind::i8 tensor-core GEMM with fused dequant: K >= 128;
                       BL_W_I8 rows need ldw % 16 == 0.  Packed weights are decoded
                       inside the GEMM for M <= 512 and unpacked into the workspace
                       beyond; with fewer 128 x 256 output tiles than 148, K is split
                       across CTAs and the int32 partials [split, M, N] go to the
                       workspace (one more launch sums them; exact) */
} bl_path;

/* Flags OR'd into the `path` argument of bl_linear_ex and bl_linear_acc_ex,
 * and passed as `flags` to bl_linear_group.
 *
 * BL_FLAG_STATIC_WEIGHTS: the caller guarantees that W is not written by any
 * kernel that may still be running when the call is issued (for instance
 * weights quantized once and only read while decoding).  The GEMV and the
 * swapped tensor-core GEMM are launched with programmatic dependent launch in
 * every case, so their prologue overlaps the previous kernel on the stream;
 * with this flag the swapped GEMM also starts copying W before that kernel has
 * finished (its weights have a producer of their own), and waits for it only
 * before reading X and writing Y.  The decode GEMV copies X first either way
 * (a weight copy issued ahead of X was measured to delay it).  Results are
 * identical with and without the flag; a call that breaks the guarantee may
 * read stale weights. */
#define BL_FLAG_STATIC_WEIGHTS 0x100

/* Packed row stride in bytes: ceil(K/5) rounded up to a multiple of 16. */
int64_t bl_pack5_ldp(int64_t K);

/* Bytes of `ws` that bl_absmean and bl_quantize_weights* need (16384). */
size_t bl_quantize_weights_workspace_size(int64_t N, int64_t K);

/* Step 1 of the weight quantization: beta = (1/n) sum |W| + eps ("the bytes",
 * absmean equation), one scalar for the whole tensor ("global beta", section
 * "autograd on a byte-graph").
 *   W        [N, K] float32, contiguous, 4-byte aligned (16 bytes for full speed).
 *   eps      finite, > 0.
 *   beta_dev one float32 on the device: receives beta.
 *   ws       >= bl_quantize_weights_workspace_size(N, K) bytes (16 KB), 256-byte
 *            aligned, ZERO-FILLED before its first use (e.g. cudaMemsetAsync);
 *            every call leaves it zero-filled again, so a workspace is cleared
 *            once and reused.  Calls sharing one workspace must not overlap on
 *            the GPU (issue them on one stream).  A workspace found not cleared
 *            is reported as BL_ERR_WORKSPACE by bl_sync_status.
 * A non-finite weight sets BL_ERR_NONFINITE in the status word. */
bl_status bl_absmean(const float* W, int64_t N, int64_t K, float eps, float* beta_dev, void* ws,
                     size_t ws_bytes, cudaStream_t stream);

/* Step 2: W_q = clip(round(W / beta), -1, 1) with beta read from beta_dev
 * ("the bytes").  W [N, K] float32 contiguous -> Wq [N, K] int8 contiguous. */
bl_status bl_ternarize(const float* W, int64_t N, int64_t K, const float* beta_dev, int8_t* Wq,
                       cudaStream_t stream);

/* Steps 2 and 3 fused: the codes of bl_ternarize written straight into the
 * packed format, Wp [N, ldp] uint8 (ldp % 16 == 0, ldp >= ceil(K/5), Wp 16-byte
 * aligned).  Equals bl_ternarize followed by bl_pack. */
bl_status bl_ternarize_pack5(const float* W, int64_t N, int64_t K, const float* beta_dev,
                             uint8_t* Wp, int64_t ldp, cudaStream_t stream);

/* bl_absmean then bl_ternarize: the whole absmean ternarization, one trit per
 * byte.  Wq [N, K] int8 contiguous; beta_dev receives beta (no host sync).
 * Errors: BL_ERR_INVALID_ARG, BL_ERR_WORKSPACE, BL_ERR_CUDA; a non-finite
 * weight sets BL_ERR_NONFINITE in the status word (codes are then unspecified). */
bl_status bl_quantize_weights(const float* W, int64_t N, int64_t K, float eps, int8_t* Wq,
                              float* beta_dev, void* ws, size_t ws_bytes, cudaStream_t stream);

/* bl_absmean then bl_ternarize_pack5: the same codes, packed five per byte,
 * without the int8 round trip. */
bl_status bl_quantize_weights_pack5(const float* W, int64_t N, int64_t K, float eps,
                                    uint8_t* Wp, int64_t ldp, float* beta_dev, void* ws,
                                    size_t ws_bytes, cudaStream_t stream);

/* int8 trits [N, K] (contiguous) -> packed [N, ldp] (format BL_W_PACK5).
 * Codes outside {-1,0,1} are a caller error (the byte is then unspecified). */
bl_status bl_pack(const int8_t* Wq, int64_t N, int64_t K, uint8_t* Wp, int64_t ldp,
                  cudaStream_t stream);

/* packed [N, ldp] -> int8 trits [N, K] (contiguous); the inverse of bl_pack. */
bl_status bl_unpack(const uint8_t* Wp, int64_t N, int64_t K, int64_t ldp, int8_t* Wq,
                    cudaStream_t stream);

/* Per-row absmax int8 quantization ("the bytes"; per-token scales, section
 * "attention, as graph ops").
 *   X  [M, K] float32, contiguous.   Xq [M, K] int8, contiguous.   s [M] float32.
 * Rows are independent: row m's outputs depend on row m of X only. */
bl_status bl_quantize_act(const float* X, int64_t M, int64_t K, float eps, int8_t* Xq,
                          float* s, cudaStream_t stream);

/* RMSNorm fused into the per-row activation quantization: the input of a
 * BitLinear in a pre-norm block ("ultragraph-1bit 0.12.0" (PyPI): "x = x +
 * mha(norm1(x))"), with RMSNorm(x) = x / sqrt((1/K) sum_k x_k^2 + eps_norm) * g
 * ("ultragraph -- when the graph is the 1-bit LLM, part 2", section "attention,
 * as graph ops"), then s and x_q of bl_quantize_act on the normalized row.
 *   X [M, K] float32 contiguous, g [K] float32 (the gain), 1 <= K <= 49152.
 *   eps_norm, eps: finite, > 0 (the norm's and the quantizer's).
 *   Xq [M, K] int8, s [M] float32 (outputs).
 * The mean of squares is exact: the sum of the float32 squares is formed
 * exactly and rounded once to float64, divided by K in float64 and rounded to
 * float32; + eps_norm, sqrt, x / r and * g are float32 IEEE steps.  One read of
 * X; rows are independent. */
bl_status bl_rmsnorm_quantize_act(const float* X, int64_t M, int64_t K, const float* g, float eps_norm, float eps,
                                  int8_t* Xq, float* s, cudaStream_t stream);

/* Bytes of `ws` that bl_linear needs for this shape and format (0 for shapes
 * that take the decode GEMV: ws may then be NULL). */
size_t bl_linear_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f);

/* Bytes of `ws` that bl_linear_ex needs with kernel path `path` pinned. */
size_t bl_linear_ex_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path);

/* The BitLinear forward: Y = (X_q W_q^T)(s beta) [+ bias], X_q and s computed
 * from X inside the call (deployed-path equation).
 *   X        [M, K] float32 contiguous.  M may be 0 (nothing is launched).
 *   W        weights in format f, [N, ldw] (BL_W_I8: ldw >= K; BL_W_PACK5:
 *            ldw % 16 == 0, ldw >= ceil(K/5), W 16-byte aligned).
 *   beta_dev the tensor's beta on the device (from bl_quantize_weights*).
 *   bias     [N] float32 or NULL.
 *   Y        [M, N] float32 contiguous output.
 *   ws       >= bl_linear_workspace_size(M, N, K, f) bytes, 256-byte aligned
 *            (NULL when that size is 0). */
bl_status bl_linear(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f, int64_t N,
                    int64_t ldw, const float* beta_dev, const float* bias, float eps, float* Y,
                    void* ws, size_t ws_bytes, cudaStream_t stream);

/* The BitLinear forward pass, steps 1-6 in one call: the weight tensor's beta
 * and codes (as bl_quantize_weights / bl_quantize_weights_pack5), then
 * Y = (X_q W_q^T)(s beta) [+ bias] (as bl_linear) -- the layer of "ultragraph
 * -- when the graph is the 1-bit LLM, part 2", sections "the bytes" and
 * "autograd on a byte-graph", where every forward quantizes both operands.
 *   X        [M, K] float32 contiguous (16-byte aligned for the one-launch path).
 *   W        [N, K] float32 contiguous.
 *   f, Wout  the codes written out: BL_W_PACK5 [N, ldo] (ldo % 16 == 0,
 *            ldo >= ceil(K/5), 16-byte aligned) or BL_W_I8 [N, K] (ldo == K).
 *   beta_dev receives beta; bias [N] float32 or NULL; Y [M, N] float32.
 *   eps      the epsilon of both quantizers.
 *   ws       >= bl_bitlinear_forward_workspace_size(M, N, K, f) bytes, 256-byte
 *            aligned, zero-filled before its first use (as for
 *            bl_quantize_weights); calls sharing it must not overlap.
 * For M <= 4 (decode) and tensors of 2^20+ weights with K % 4 == 0 and
 * M*K*4 <= 48 KB, one cooperative launch reads W once and computes everything;
 * other shapes run bl_quantize_weights* and bl_linear.  Results are identical
 * either way.  Errors as for those two calls. */
size_t bl_bitlinear_forward_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f);
bl_status bl_bitlinear_forward(const float* X, int64_t M, int64_t K, const float* W, bl_wfmt f,
                               int64_t N, float eps, void* Wout, int64_t ldo, float* beta_dev,
                               const float* bias, float* Y, void* ws, size_t ws_bytes,
                               cudaStream_t stream);

/* bl_linear with the kernel path pinned (BL_PATH_*, optionally OR'd with
 * BL_FLAG_STATIC_WEIGHTS); BL_ERR_UNSUPPORTED when the pinned path cannot take
 * the shape.  Results are identical across paths. */
bl_status bl_linear_ex(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f,
                       int64_t N, int64_t ldw, const float* beta_dev, const float* bias,
                       float eps, float* Y, void* ws, size_t ws_bytes, int path,
                       cudaStream_t stream);

/* The kernel path bl_linear_ex(..., path) would run for this shape (BL_PATH_*),
 * or -1 if that path cannot take it; *launches (if not NULL) receives the number
 * of kernel launches the call makes.  Assumes contiguous weight rows (ldw = K
 * for BL_W_I8, bl_pack5_ldp(K) for BL_W_PACK5).  Host-only, no CUDA call. */
int bl_linear_plan(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path, int* launches);

/* The contraction alone: acc[m,n] = sum_k Xq[m,k] * W_q[n,k] in int32, from
 * pre-quantized activations Xq [M, K] int8 contiguous; acc [M, N] int32.
 * (The integer product x_q W_q^T of the deployed-path equation.)  Needs no
 * workspace: on the tensor cores packed weights are then decoded inside the
 * GEMM at any M and K is not split. */
bl_status bl_linear_acc(const int8_t* Xq, int64_t M, int64_t K, const void* W, bl_wfmt f,
                        int64_t N, int64_t ldw, int32_t* acc, cudaStream_t stream);

/* bl_linear_acc with the kernel path pinned; ws as for bl_linear (may be NULL
 * when bl_linear_acc_workspace_size returns 0). */
size_t bl_linear_acc_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path);
bl_status bl_linear_acc_ex(const int8_t* Xq, int64_t M, int64_t K, const void* W, bl_wfmt f,
                           int64_t N, int64_t ldw, int32_t* acc, void* ws, size_t ws_bytes,
                           int path, cudaStream_t stream);

/* One call of bl_linear_group: the arguments of bl_linear, minus the workspace. */
typedef struct {
  const float* X;        /* [M, K] float32 */
  int64_t M, K;
  const void* W;         /* weights in format f, [N, ldw] */
  int64_t N, ldw;
  bl_wfmt f;
  float eps;
  const float* beta_dev;
  const float* bias;     /* [N] or NULL */
  float* Y;              /* [M, N] float32 */
} bl_linear_call;

/* Bytes of `ws` that bl_linear_group needs for these calls (0 when every call
 * takes the decode GEMV). */
size_t bl_linear_group_workspace_size(const bl_linear_call* calls, int count);

/* Several independent BitLinear forwards (deployed-path equation, as bl_linear)
 * in as few launches as possible: the calls that take the decode GEMV (packed
 * weights, M <= 4) run in one launch per M, up to four problems each, so their
 * weight streams share one grid (for instance the projections of one decode
 * step that read the same or separate activations); the other calls run as
 * bl_linear would, each with its own part of `ws`.  Results are bit-identical
 * to `count` bl_linear calls.  The calls must be independent: no call's Y may
 * overlap another call's X, W, beta, bias or Y.  `flags`: 0 or
 * BL_FLAG_STATIC_WEIGHTS.  Every call is validated before anything launches;
 * errors as for bl_linear. */
bl_status bl_linear_group(const bl_linear_call* calls, int count, int flags, void* ws, size_t ws_bytes,
                          cudaStream_t stream);

/* The host buffers of one call of bl_linear_group_host. */
typedef struct {
  const float* X_host;   /* [M, K] float32 rows in host memory, contiguous */
  float* Y_host;         /* [M, N] float32 in host memory, contiguous */
} bl_host_io;

/* bl_linear_group with the activations read from, and the results written to,
 * host memory (same equation and results as bl_linear_group).  Enqueued on
 * `stream`, in this order, with no host synchronization:
 *   1. io[i].X_host (M*K floats) is moved into calls[i].X, which serves as the
 *      call's device staging buffer (the library overwrites it);
 *   2. the calls run as bl_linear_group(calls, count, flags, ws, ws_bytes);
 *   3. the results (M*N floats per call) land in io[i].Y_host.
 * The caller synchronizes `stream` before it reads Y_host or reuses X_host.
 * How the bytes move:
 *   - Host memory that is page-locked and mapped into the device's address space
 *     (cudaHostAlloc / cudaMallocHost, or cudaHostRegister'd memory, on a system
 *     with unified addressing): the activations, up to 4 MiB per call of this
 *     function, are read over the bus by a kernel of the library (no copy-engine
 *     hand-off between kernels), and a call on the decode GEMV stores its results
 *     straight into Y_host (its calls[i].Y is then left unwritten).
 *   - Otherwise (pageable memory, larger inputs, other paths): copies on
 *     `stream`; those of consecutive calls whose host ranges and device ranges
 *     both follow one another end to end are merged into one transfer.  From
 *     pageable memory the CUDA runtime stages the copies and they may return
 *     only once done.
 * Ownership: all buffers stay the caller's.
 * Errors: as bl_linear_group; BL_ERR_INVALID_ARG also for a NULL `io` (count >
 * 0) or a NULL host pointer of a call with M > 0.  Every call is validated
 * before anything is enqueued; BL_ERR_CUDA if a copy or launch cannot be
 * enqueued (work enqueued before it stays enqueued). */
bl_status bl_linear_group_host(const bl_linear_call* calls, const bl_host_io* io, int count, int flags,
                               void* ws, size_t ws_bytes, cudaStream_t stream);

/* Size of the scratch array built into the library for bl_linear_noalloc. */
#define BL_LINEAR_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* bl_linear for callers that cannot allocate device memory at all: a plugin or
 * custom-op interface that hands the library only its input and output buffers
 * and owns every allocation under a fixed memory plan, or a latency-critical
 * loop where cudaMalloc (which may synchronize the whole device) is not allowed.
 * The paper has no counterpart to this entry point: it is a deployment
 * convenience of this library.
 *
 * Same arguments and results as bl_linear, minus the workspace.  The scratch
 * (quantized activations and row scales) is a static device array of
 * BL_LINEAR_NOALLOC_SCRATCH_BYTES that every GPU loading the library holds until
 * the process exits.  Nothing is allocated: no cudaMalloc, cudaFree or
 * allocating library routine is called.
 *   - Shapes whose bl_linear_workspace_size(M, N, K, f) exceeds the array run
 *     the tensor-core GEMM without its K split (whose partials are most of
 *     that workspace) if the rest fits; otherwise they are rejected with
 *     BL_ERR_WORKSPACE before anything is launched.
 *   - The first call on each device looks up the array's device address with
 *     cudaGetSymbolAddress (with that device current); make that first call
 *     before any stream capture.
 *   - All calls on a device share the one array and it keeps the last call's
 *     contents: calls that overlap on the GPU (other streams, other host
 *     threads) race on it, so issue them in order on one stream.  Every scratch
 *     byte a call reads is written earlier in the same call, so nothing needs
 *     clearing between calls. */
bl_status bl_linear_noalloc(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f,
                            int64_t N, int64_t ldw, const float* beta_dev, const float* bias,
                            float eps, float* Y, cudaStream_t stream);

/* ---- straight-through backward --------------------------------------------
 * "ultragraph -- when the graph is the 1-bit LLM, part 2", section "autograd on
 * a byte-graph, and the straight-through lie": the backward of y = (x_q W_q^T)
 * (s beta) + b treats the quantizers and the per-row scale as the identity, so
 *     dX = dY W  [M, K],   dW = dY^T X  [N, K],   db = sum over rows of dY  [N],
 * with W the float32 master weights [N, K] and X the float32 input [M, K].
 *
 * Bytes of `ws` that bl_linear_backward needs (float32 hi/lo splits of the
 * operands of one product at a time). */
size_t bl_linear_backward_workspace_size(int64_t M, int64_t N, int64_t K);

/* The three gradients; any of dX, dW, db may be NULL to skip it.
 *   dY [M, N], X [M, K], W [N, K], dX [M, K], dW [N, K], db [N]: float32,
 *   contiguous, 4-byte aligned.  X may be NULL when dW is, W when dX is.
 *   ws  >= bl_linear_backward_workspace_size(M, N, K) bytes, 256-byte aligned
 *       (may be NULL when dX and dW are both NULL).
 * The products run on the tensor cores (tcgen05 kind::tf32, float32
 * accumulators) with every float32 operand split into two tf32 parts, a = a_hi
 * + a_lo, and the three products a_hi b_hi + a_hi b_lo + a_lo b_hi: each
 * product is then within about 3 * 2^-22 |a b| of the exact one, and an output
 * is within (3 * 2^-22 + (n + 1) 2^-24) sum |a b| of the exact sum, n being
 * the 3 * ceil(Kc / 8) accumulator updates over the contraction length Kc.
 * db is summed in float64 and rounded once.  M == 0 launches nothing. */
bl_status bl_linear_backward(const float* dY, const float* X, const float* W, int64_t M, int64_t N, int64_t K,
                             float* dX, float* dW, float* db, void* ws, size_t ws_bytes, cudaStream_t stream);

/* ---- deployed checkpoint ---------------------------------------------------
 * "ultragraph-1bit 0.12.0" (PyPI), section "A whole ternary GPT": a deployed
 * checkpoint stores the ternary weights at five per byte (~1.6 bits each) plus
 * the float32 pieces, and a model loaded from it computes exactly what the
 * model that wrote it computes, straight from the stored bytes.  File layout
 * (little-endian, no padding):
 *   "BLT5", version u32 = 1, count u32, reserved u32 = 0, then per layer:
 *   name_len u32 (<= 255), name bytes, N u64, K u64, flags u32 (bit 0: bias),
 *   beta u32 (float32 bits), the packed rows (N * ceil(K/5) bytes: BL_W_PACK5
 *   rows without their padding), [bias: N float32].
 * These calls are synchronous: they wait for the work queued on `stream`, copy
 * through host staging buffers (at most 64 MB, malloc'd and freed inside the
 * call; no device memory is allocated) and return when the copies are done.
 * A file that cannot be opened, written or read, that is truncated or has
 * trailing bytes, or that holds a byte above 242 in its packed rows gives
 * BL_ERR_IO; a failed save removes the partial file. */
typedef struct {
  const char* name;        /* NUL-terminated, at most 255 bytes; NULL = "" */
  int64_t N, K;
  const uint8_t* Wp;       /* device, packed trits [N, ldp] (BL_W_PACK5) */
  int64_t ldp;             /* >= ceil(K/5) */
  const float* beta_dev;   /* device, the tensor's beta */
  const float* bias_dev;   /* device [N] float32, or NULL (no bias stored) */
} bl_deployed_layer;

/* Writes `count` layers to `path` (replacing it). */
bl_status bl_save_deployed(const char* path, const bl_deployed_layer* layers, int count, cudaStream_t stream);

/* The number of layers in the checkpoint at `path` (the whole file is checked). */
bl_status bl_deployed_count(const char* path, int* count);

/* Layer `index`'s shape, whether it stores a bias, and its name (copied into
 * `name`, at most name_cap - 1 bytes and a NUL; NULL to skip).  Host only. */
bl_status bl_deployed_layer_info(const char* path, int index, int64_t* N, int64_t* K, int* has_bias, char* name,
                                 size_t name_cap);

/* Layer `index` into device buffers: Wp [N, ldp] (ldp % 16 == 0, >= ceil(K/5),
 * 16-byte aligned; bytes past ceil(K/5) in each row are set to 121, five zero
 * trits, exactly as bl_pack writes them), beta_dev (one float32, bit for bit),
 * bias_dev ([N] float32; NULL to skip; BL_ERR_INVALID_ARG if the layer has no
 * bias). */
bl_status bl_load_deployed_layer(const char* path, int index, uint8_t* Wp, int64_t ldp, float* beta_dev,
                                 float* bias_dev, cudaStream_t stream);

/* Synchronizes `stream`, then reads and clears this device's status word:
 * BL_ERR_DEVICE_TIMEOUT or BL_ERR_NONFINITE if a kernel recorded one, BL_ERR_CUDA
 * if the stream reports an error, else BL_OK. */
bl_status bl_sync_status(cudaStream_t stream);

/* Self-test of the device timeout path: one thread waits, with the bounded
 * wait every kernel of this library uses, on an mbarrier phase that nothing
 * completes, and gives up after `limit_ns` nanoseconds of %globaltimer
 * (1000 <= limit_ns <= 10^9, else BL_ERR_INVALID_ARG); it records the timeout
 * in the status word as any kernel does, so the next bl_sync_status returns
 * BL_ERR_DEVICE_TIMEOUT (and clears it).  Nothing faults or hangs. */
bl_status bl_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream);

/* A static, human-readable name for a status code. */
const char* bl_status_string(bl_status s);

#ifdef __cplusplus
}
#endif

#endif /* BITLINEAR_H_ */
