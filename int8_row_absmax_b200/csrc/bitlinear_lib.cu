// C ABI of the BitLinear library (declared in include/bitlinear.h).
//
// Host-side argument checks, workspace carving and kernel dispatch.  Every
// step of the computation runs in the kernels included below; there is no CPU
// fallback.  One translation unit, so the per-device status word is a single
// symbol without relocatable device code.
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <vector>

#include <cuda_runtime.h>

#include "bitlinear.h"
#include "common.cuh"
#include "weight_quant.cuh"
#include "weight_fused.cuh"
#include "pack.cuh"
#include "act_quant.cuh"
#include "linear_simt.cuh"
#include "gemv_pack5.cuh"
#include "gemm_tc.cuh"
#include "gemm_swap.cuh"
#include "deployed_io.cuh"
#include "ste_backward.cuh"
#include "rmsnorm_quant.cuh"
#include "host_io.cuh"

namespace bl {
namespace {

constexpr size_t kWsAlign = 256;
constexpr int kPathMask = 0xFF;   // the BL_PATH_* bits of a `path` argument (flags above)

size_t align_up(size_t v) { return (v + kWsAlign - 1) / kWsAlign * kWsAlign; }

bool eps_ok(float eps) { return std::isfinite(eps) && eps > 0.f; }

bool is_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms > 0 ? sms : 148;
}

unsigned grid_for(int64_t work, int per_block, int max_blocks_per_sm = 8) {
  int64_t g = ceil_div(work, per_block);
  const int64_t cap = int64_t(num_sms()) * max_blocks_per_sm;
  if (g > cap) g = cap;
  return unsigned(g < 1 ? 1 : g);
}

// Per-row activation quantization: the single-pass register kernel when the row
// fits (and is 16-byte aligned), else the two-pass kernel.
void launch_act_quant(const float* X, int64_t M, int64_t K, float eps, int8_t* Xq, int64_t ldq,
                      float* s, cudaStream_t st) {
  const bool vec = (K % 4) == 0 && (reinterpret_cast<uintptr_t>(X) % 16) == 0 &&
                   (reinterpret_cast<uintptr_t>(Xq) % 4) == 0 && (ldq % 4) == 0;
  const int64_t per_thread = ceil_div(K / 4, kActThreads);
  const unsigned g = unsigned(M);
  if (vec && per_thread <= 1) act_quant_reg_kernel<1><<<g, kActThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else if (vec && per_thread <= 2) act_quant_reg_kernel<2><<<g, kActThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else if (vec && per_thread <= 4) act_quant_reg_kernel<4><<<g, kActThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else if (vec && per_thread <= 8) act_quant_reg_kernel<8><<<g, kActThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else if (vec && per_thread <= 16) act_quant_reg_kernel<16><<<g, kActThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else act_quant_kernel<<<g, kActThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
}

bl_status launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

bl_status check_weights_args(const float* W, int64_t N, int64_t K, const void* out) {
  if (!W || !out || N < 1 || K < 1) return BL_ERR_INVALID_ARG;
  if (N > (int64_t(1) << 40) / K) return BL_ERR_INVALID_ARG;
  if (!is_aligned(W, 4)) return BL_ERR_ALIGNMENT;
  return BL_OK;
}

// a1: beta of a weight tensor into beta_dev, one launch.
bl_status launch_absmean(const float* W, int64_t n, float eps, float* beta_dev, void* ws,
                         cudaStream_t st) {
  auto* acc = static_cast<AbsAccum*>(ws);
  if (cudaFuncSetAttribute(absmean_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kAbsSmem) !=
      cudaSuccess)
    return BL_ERR_CUDA;
  // one persistent CTA per SM, fewer when there are fewer 32 KB chunks
  const int64_t chunks = ceil_div(n, kAbsChunkFloats);
  int grid = int(chunks < num_sms() ? (chunks < 1 ? 1 : chunks) : num_sms());
  if (grid > kAbsMaxCtas) grid = kAbsMaxCtas;
  absmean_kernel<<<grid, kAbsThreads, kAbsSmem, st>>>(W, n, eps, acc, beta_dev);
  return launch_status();
}

// Whether the single-pass quantizer applies: large enough to pay for its extra
// launches, 16-byte rows for the bulk copies, column index within 17 bits.
bool fused_shape(int64_t N, int64_t K) { return N * K >= kFusedMinN && K % 4 == 0 && K <= 131072; }

// a1-a3 in one read of W: one cooperative launch (all CTAs resident, for the
// kernel's two grid barriers); with M > 0 rows of X also a4-a6 (the BitLinear
// forward) in the same launch.  Returns BL_ERR_UNSUPPORTED, with nothing
// launched, when the device cannot hold the grid at once.
template <bool kPacked, int kM>
const void* wquant_fn() {
  return reinterpret_cast<const void*>(wquant_kernel<kPacked, kM>);
}
const void* wquant_pick(bool packed, int M) {
  switch (M) {
    case 0: return packed ? wquant_fn<true, 0>() : wquant_fn<false, 0>();
    case 1: return packed ? wquant_fn<true, 1>() : wquant_fn<false, 1>();
    case 2: return packed ? wquant_fn<true, 2>() : wquant_fn<false, 2>();
    case 3: return packed ? wquant_fn<true, 3>() : wquant_fn<false, 3>();
    default: return packed ? wquant_fn<true, 4>() : wquant_fn<false, 4>();
  }
}

bl_status launch_wquant_fused(const float* W, int64_t N, int64_t K, float eps, void* out,
                              int64_t ldo, bool packed, float* beta_dev, void* ws,
                              cudaStream_t st, int64_t M = 0, const float* X = nullptr,
                              const float* bias = nullptr, float* Y = nullptr) {
  WqArgs a;
  a.W = W;
  a.N = N;
  a.K = K;
  a.eps = eps;
  a.out = out;
  a.ldo = ldo;
  a.acc = static_cast<AbsAccum*>(ws);
  a.yacc = reinterpret_cast<int*>(static_cast<char*>(ws) + kFuListOff);
  a.list = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + kFuListOff +
                                                 fused_acc_bytes(M, N));
  a.beta_out = beta_dev;
  a.X = X;
  a.bias = bias;
  a.Y = Y;
  const int64_t ngroups = N * ceil_div(K, 20);
  const int64_t nch = ceil_div(ngroups, kFuGroups);
  const int stages = M > 0 ? kFuStagesFwd : kFuStages;
  a.xf_off = uint32_t(stages) * kFuStageBytes;
  const int smem = int(a.xf_off + uint32_t(M * K * 4));
  const void* fn = wquant_pick(packed, int(M));
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BL_ERR_CUDA;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, fn, kAbsThreads, smem) != cudaSuccess)
    return BL_ERR_CUDA;
  int grid = num_sms() * per_sm;
  if (grid > kAbsMaxCtas) grid = kAbsMaxCtas;
  if (int64_t(grid) > nch) grid = int(nch);
  if (grid < 1) return BL_ERR_UNSUPPORTED;
  a.cap_w = int(fused_cap_w(ngroups, grid));
  a.stride = chunk_stride(nch, grid);
  const int64_t gpr = ceil_div(K, 20);
  a.gpr_magic = gpr > 1 ? uint32_t(((uint64_t(1) << 32) + uint64_t(gpr) - 1) / uint64_t(gpr)) : 0u;
  void* args[] = {&a};
  const cudaError_t e = cudaLaunchCooperativeKernel(fn, grid, kAbsThreads, args, size_t(smem), st);
  if (e == cudaErrorCooperativeLaunchTooLarge) {
    (void)cudaGetLastError();
    return BL_ERR_UNSUPPORTED;
  }
  return e == cudaSuccess ? BL_OK : BL_ERR_CUDA;
}

// Whether the forward can run inside the single-pass launch.
bool fused_forward_ok(int64_t M, int64_t N, int64_t K, const float* X, const float* W) {
  return M >= 1 && M <= kFwdMaxM && fused_shape(N, K) && N < (int64_t(1) << 31) &&
         uint64_t(M * K * 4) <= kFwdXBytesMax && is_aligned(X, 16) && is_aligned(W, 16);
}

bl_status check_ws(const void* ws, size_t ws_bytes, size_t need) {
  if (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < need) return BL_ERR_WORKSPACE;
  return BL_OK;
}

// ---- linear --------------------------------------------------------------
// Row stride of the swapped GEMM's decode-order codes: whole 128-byte atoms.
int64_t swap_ldx(int64_t K) { return round_up(dorder_len(K), 128); }

struct LinWs {
  int64_t ldx, ldk;
  size_t xq_off, s_off, wq_off, tc_off, total;
};
// X_q [M, ldx] and s [M]; with `unpacked_w`, an int8 copy of the packed weights
// [N, ldk] for the tensor-core path; then `tc_bytes` for the tensor-core GEMM's
// K-split partials.  With `dorder`, X_q rows are in the decode order of the
// swapped GEMM (whole packed words: dorder_len(K) bytes).
LinWs lin_layout(int64_t M, int64_t K, int64_t N = 0, bool unpacked_w = false, size_t tc_bytes = 0,
                 bool dorder = false) {
  LinWs l;
  l.ldx = dorder ? swap_ldx(K) : round_up(K, 16);
  l.ldk = round_up(K, 16);
  l.xq_off = 0;
  l.s_off = align_up(size_t(M) * size_t(l.ldx));
  l.wq_off = l.s_off + align_up(size_t(M) * 4 + 4);
  l.tc_off = l.wq_off + (unpacked_w ? align_up(size_t(N) * size_t(l.ldk)) : 0);
  l.total = l.tc_off + tc_bytes;
  return l;
}

bl_status check_w(const void* W, bl_wfmt f, int64_t K, int64_t ldw) {
  if (!W) return BL_ERR_INVALID_ARG;
  if (f == BL_W_I8) {
    if (ldw < K) return BL_ERR_INVALID_ARG;
  } else if (f == BL_W_PACK5) {
    if (ldw < ceil_div(K, 5)) return BL_ERR_INVALID_ARG;
    if (ldw % 16 != 0 || !is_aligned(W, 16)) return BL_ERR_ALIGNMENT;
  } else {
    return BL_ERR_INVALID_ARG;
  }
  return BL_OK;
}

bl_status check_shape(int64_t M, int64_t K, int64_t N) {
  if (M < 0 || N < 1 || K < 1 || K > kMaxK) return BL_ERR_INVALID_ARG;
  if (M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1) return BL_ERR_INVALID_ARG;
  return BL_OK;
}

// Resolve the kernel path for a linear call; -1 when the pinned path cannot run it.
// `fused_quant`: bl_linear (X in float32) rather than bl_linear_acc (X_q given).
// Packed weights are decoded inside the tensor-core GEMM for up to this many
// 128-row tiles; beyond, they are unpacked to int8 once and the GEMM reads those.
constexpr int64_t kTcDecodeMaxTilesM = 4;
bool tc_unpack(int64_t M, bl_wfmt f) { return f == BL_W_PACK5 && ceil_div(M, int64_t(kTcBM)) > kTcDecodeMaxTilesM; }

// K split of the tensor-core GEMM: with fewer 128 x 256 tiles than SMs, each
// tile's K is cut into `split` ranges of whole 640-wide chunks (at most
// kTcMaxSplit), whose int32 partial tiles [split, M, N] live in the workspace;
// tc_reduce_kernel sums them (one more launch).
// The split is planned for B200's 148 SMs (a fixed figure, so that planning
// and workspace sizes need no device query; the grid is still capped by the
// device's own SM count).
constexpr int64_t kTcSplitSms = 148;
struct TcSplit {
  int64_t tiles;
  int split;
  size_t bytes;
};
// Few-row packed layers (5 <= M <= 128) run the swapped GEMM: W rows are the
// MMA's M side, X rows its N side (gemm_swap.cuh).
bool tc_swap(int64_t M, bl_wfmt f) { return f == BL_W_PACK5 && M >= 1 && M <= kSwMaxNp; }

TcSplit tc_split(int64_t M, int64_t N, int64_t K, bl_wfmt f) {
  TcSplit r;
  int64_t nch;
  if (tc_swap(M, f)) {   // 128-row W tiles, K chunks of four 160-trit blocks
    r.tiles = ceil_div(N, int64_t(kSwBM));
    nch = ceil_div(K, int64_t(kSwBoxKb * kSwBK));
  } else {
    r.tiles = ceil_div(M, int64_t(kTcBM)) * ceil_div(N, int64_t(kTcBN));
    nch = ceil_div(ceil_div(K, int64_t(kTcBK)), int64_t(kTcChunk));
  }
  int64_t sp = kTcSplitSms / (r.tiles > 0 ? r.tiles : 1);
  if (sp > nch) sp = nch;
  if (sp > kTcMaxSplit) sp = kTcMaxSplit;
  r.split = int(sp < 1 ? 1 : sp);
  r.bytes = r.split > 1 ? align_up(size_t(r.split) * size_t(M) * size_t(N) * 4) : 0;
  return r;
}
// AUTO: the swapped tensor-core GEMM from M = 4 for packed weights (measured
// faster than the dp4a GEMV there at K = 2560 .. 8192), the tensor cores from
// M = 5 for one trit per byte.
constexpr int64_t kSwMinM = 4;
constexpr int64_t kTcMinM = 5;

// Whether the tensor-core path can take the shape: K at least one 128-byte K
// block, and for one-trit-per-byte weights a TMA-able row stride.
bool tc_feasible(int64_t M, int64_t N, int64_t K, bl_wfmt f, int64_t ldw, const void* W) {
  if (M < 1 || N < 1 || K < kTcBK) return false;
  if (f == BL_W_I8) return ldw % 16 == 0 && (W == nullptr || is_aligned(W, 16));
  return f == BL_W_PACK5;
}

int resolve_path(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path, int* launches,
                 bool fused_quant = true, int64_t ldw = -1, const void* W = nullptr) {
  const int64_t ldp = round_up(ceil_div(K, 5), 16);
  if (ldw < 0) ldw = f == BL_W_PACK5 ? ldp : K;   // contiguous rows unless told otherwise
  const bool gemv_ok = f == BL_W_PACK5 && M >= 1 && gemv_feasible(M, N, K, ldp);
  const bool tc_ok = tc_feasible(M, N, K, f, ldw, W);
  int p = path;
  if (p == BL_PATH_AUTO)
    p = (M >= (f == BL_W_PACK5 ? kSwMinM : kTcMinM) && tc_ok) ? BL_PATH_TC : (gemv_ok ? BL_PATH_GEMV : BL_PATH_SIMT);
  int n = 0;
  if (p == BL_PATH_SIMT) {
    n = fused_quant ? 2 : 1;  // act_quant + contraction
  } else if (p == BL_PATH_GEMV) {
    if (!gemv_ok) return -1;
    n = 1;                    // quantization fused into the GEMV
  } else if (p == BL_PATH_TC) {
    if (!tc_ok) return -1;
    // [act_quant,] [unpack,] GEMM [, K-split reduction]
    n = (fused_quant ? 2 : 1) + (tc_unpack(M, f) ? 1 : 0) + (tc_split(M, N, K, f).split > 1 ? 1 : 0);
  } else {
    return -1;
  }
  if (launches) *launches = M == 0 ? 0 : n;
  return p;
}

// ---- tensor maps (driver entry point, so the library does not link libcuda) ---
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D int8 [outer, inner] matrix with row stride `ld` bytes, 128-byte swizzled
// boxes of {128, box_rows}; out-of-range elements read as zero.
bool make_map_i8(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld,
                 int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(outer)};
  const cuuint64_t strides[1] = {cuuint64_t(ld)};
  const cuuint32_t box[2] = {cuuint32_t(kTcBK), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed W [N, ldp] bytes as 128-byte x rows boxes with the 128-byte swizzle
// (the decoder warps' reads of four rows then spread over the banks);
// out-of-range bytes are 0 (they only meet zero X columns).
bool make_map_packed(CUtensorMap* map, const void* base, int64_t ldp, int64_t N, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(ldp), cuuint64_t(N)};
  const cuuint64_t strides[1] = {cuuint64_t(ldp)};
  const cuuint32_t box[2] = {128u, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// float32 [outer, inner] (row stride ld floats, a multiple of 4) as 128-byte
// swizzled boxes of {32, box_rows}; out-of-range elements read as zero.
bool make_map_f32(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(inner), cuuint64_t(outer)};
  const cuuint64_t strides[1] = {cuuint64_t(ld) * 4};
  const cuuint32_t box[2] = {cuuint32_t(kBwBK), cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// D [Mr, Nc] = A B^T over Kc from the hi/lo splits of A [Mr, ld] and B [Nc, ld].
bl_status run_tf32x3(const float* ahi, const float* alo, const float* bhi, const float* blo, int64_t ld, int64_t Mr,
                     int64_t Nc, int64_t Kc, float* D, cudaStream_t st) {
  BwMaps maps;
  if (!make_map_f32(&maps.a_hi, ahi, Kc, Mr, ld, kBwBM) || !make_map_f32(&maps.a_lo, alo, Kc, Mr, ld, kBwBM) ||
      !make_map_f32(&maps.b_hi, bhi, Kc, Nc, ld, kBwBN) || !make_map_f32(&maps.b_lo, blo, Kc, Nc, ld, kBwBN))
    return BL_ERR_CUDA;
  BwArgs a;
  a.Mr = Mr;
  a.Nc = Nc;
  a.Kc = Kc;
  a.D = D;
  a.tiles_m = int(ceil_div(Mr, int64_t(kBwBM)));
  a.tiles_n = int(ceil_div(Nc, int64_t(kBwBN)));
  const int64_t work = int64_t(a.tiles_m) * a.tiles_n;
  if (cudaFuncSetAttribute(gemm_tf32x3_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBwSmem) != cudaSuccess)
    return BL_ERR_CUDA;
  gemm_tf32x3_kernel<<<unsigned(work < num_sms() ? work : num_sms()), kBwThreads, kBwSmem, st>>>(maps, a);
  return launch_status();
}

// The tcgen05 GEMM on int8 X_q [M, ldx] and int8 W_q [N, ldw] (or packed W
// [N, ldw = ldp], decoded inside the kernel).
template <bool kPacked>
bl_status launch_tc(const TcMaps& maps, const TcArgs& a, bool dequant, cudaStream_t st) {
  const int64_t work = int64_t(a.tiles_m) * a.tiles_n * a.split;
  const dim3 grid(unsigned(work < num_sms() ? work : num_sms()));
  constexpr int smem = TcCfg<kPacked>::kSmem;
  constexpr int threads = TcCfg<kPacked>::kThreads;
  if (dequant) {
    if (cudaFuncSetAttribute(gemm_tc_kernel<true, kPacked>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return BL_ERR_CUDA;
    gemm_tc_kernel<true, kPacked><<<grid, threads, smem, st>>>(maps, a);
  } else {
    if (cudaFuncSetAttribute(gemm_tc_kernel<false, kPacked>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) !=
        cudaSuccess)
      return BL_ERR_CUDA;
    gemm_tc_kernel<false, kPacked><<<grid, threads, smem, st>>>(maps, a);
  }
  return launch_status();
}

bl_status run_tc(const int8_t* Xq, int64_t ldx, int64_t M, int64_t K, const void* W, int64_t ldw,
                 bool packed, int64_t N, const float* s, const float* beta, const float* bias, float* Y,
                 int32_t* acc, void* tcws, size_t tcws_bytes, cudaStream_t st) {
  if (ldx % 16 != 0 || ldw % 16 != 0 || !is_aligned(Xq, 16) || !is_aligned(W, 16))
    return BL_ERR_ALIGNMENT;
  // no workspace (tcws null): no K split
  TcSplit sp = tc_split(M, N, K, packed ? BL_W_PACK5 : BL_W_I8);
  if (!tcws) sp.split = 1;
  if (sp.tiles > (int64_t(1) << 28)) return BL_ERR_UNSUPPORTED;
  if (sp.split > 1 && (!is_aligned(tcws, kWsAlign) || tcws_bytes < sp.bytes)) return BL_ERR_WORKSPACE;
  TcMaps maps;
  if (!make_map_i8(&maps.a, Xq, K, M, ldx, kTcBM)) return BL_ERR_CUDA;
  if (packed ? !make_map_packed(&maps.b, W, ldw, N, kTcBN) : !make_map_i8(&maps.b, W, K, N, ldw, kTcBN))
    return BL_ERR_CUDA;
  TcArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.s = s;
  a.beta = beta;
  a.bias = bias;
  a.Y = Y;
  a.acc = acc;
  a.tiles_m = int(ceil_div(M, kTcBM));
  a.tiles_n = int(ceil_div(N, kTcBN));
  a.split = sp.split;
  a.part = sp.split > 1 ? static_cast<int32_t*>(tcws) : nullptr;
  const bool dq = Y != nullptr;
  const bl_status r = packed ? launch_tc<true>(maps, a, dq, st) : launch_tc<false>(maps, a, dq, st);
  if (r != BL_OK || sp.split == 1) return r;
  const int64_t work = (N % 4 == 0 ? M * (N / 4) : M * N);
  if (dq)
    tc_reduce_kernel<true><<<grid_for(work, 256), 256, 0, st>>>(a.part, sp.split, M, N, s, beta, bias, Y, nullptr);
  else
    tc_reduce_kernel<false><<<grid_for(work, 256), 256, 0, st>>>(a.part, sp.split, M, N, nullptr, nullptr, nullptr,
                                                                nullptr, acc);
  return launch_status();
}

// Packed W [N, ldp] as boxes of {128 bytes, 128 rows}, 128-byte swizzle.
bool make_map_wp128(CUtensorMap* map, const void* base, int64_t ldp, int64_t N) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cuuint64_t(ldp), cuuint64_t(N)};
  const cuuint64_t strides[1] = {cuuint64_t(ldp)};
  const cuuint32_t box[2] = {128u, cuuint32_t(kSwBM)};
  const cuuint32_t estr[2] = {1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A launch that may begin while the previous kernel on the stream finishes
// (programmatic dependent launch); the kernel waits (griddepcontrol.wait)
// before it touches what that kernel writes.
template <typename... KArgs, typename... Args>
bl_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...) == cudaSuccess ? launch_status() : BL_ERR_CUDA;
}

// X_q in decode order [M, ldx] (ldx % 128 == 0) as a 3-D tensor {128 bytes, M
// rows, ldx / 128 atoms}, boxes {128, Np, 5} (one chunk of four K blocks),
// 128-byte swizzle.
bool make_map_x3d(CUtensorMap* map, const void* base, int64_t ldx, int64_t M, int Np) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {128u, cuuint64_t(M), cuuint64_t(ldx / 128)};
  const cuuint64_t strides[2] = {cuuint64_t(ldx), 128u};
  const cuuint32_t box[3] = {128u, cuuint32_t(Np), 5u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The swapped GEMM for few-row packed layers (gemm_swap.cuh), then the K
// split's reduction when there is one.  Xd: the codes in decode order [M, ldx]
// (ldx = swap_ldx(K), bytes beyond dorder_len(K) 0).
bl_status run_swap(const int8_t* Xd, int64_t ldx, int64_t M, int64_t K, const void* W, int64_t ldw, int64_t N,
                   const float* s, const float* beta, const float* bias, float* Y, int32_t* acc, void* tcws,
                   size_t tcws_bytes, bool static_w, cudaStream_t st) {
  if (ldx % 128 != 0 || ldx < dorder_len(K) || ldw % 16 != 0 || !is_aligned(Xd, 16) || !is_aligned(W, 16))
    return BL_ERR_ALIGNMENT;
  if (M < 1 || M > kSwMaxNp) return BL_ERR_UNSUPPORTED;
  TcSplit sp = tc_split(M, N, K, BL_W_PACK5);
  if (!tcws) sp.split = 1;
  if (sp.tiles > (int64_t(1) << 28)) return BL_ERR_UNSUPPORTED;
  if (sp.split > 1 && (!is_aligned(tcws, kWsAlign) || tcws_bytes < sp.bytes)) return BL_ERR_WORKSPACE;
  const int Np = int(round_up(M, 16));
  SwMaps maps;
  if (!make_map_x3d(&maps.x, Xd, ldx, M, Np) || !make_map_wp128(&maps.wp, W, ldw, N))
    return BL_ERR_CUDA;
  SwArgs a;
  a.M = M;
  a.N = N;
  a.K = K;
  a.Np = Np;
  a.s = s;
  a.beta = beta;
  a.bias = bias;
  a.Y = Y;
  a.acc = acc;
  a.tiles = int(sp.tiles);
  a.split = sp.split;
  a.part = sp.split > 1 ? static_cast<int32_t*>(tcws) : nullptr;
  const SwLayout l = sw_layout(Np);
  if (l.nst < 1) return BL_ERR_UNSUPPORTED;
  a.nst = l.nst;
  a.xst = l.xst;
  a.lut_off = l.lut_off;
  a.x_off = l.x_off;
  a.static_w = static_w ? 1 : 0;
  a.mma_warps = sw_mma_warps(Np);
  a.a_col0 = sw_a_col0(Np);
  a.nsa = sw_a_stages(Np);
  const int64_t work = sp.tiles * sp.split;
  const dim3 grid(unsigned(work < num_sms() ? work : num_sms()));
  const bool dq = Y != nullptr;
  auto kern = dq ? gemm_swap_kernel<true> : gemm_swap_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, kSwSmemMax) != cudaSuccess)
    return BL_ERR_CUDA;
  bl_status r = launch_pdl(kern, grid, dim3(kSwThreads), size_t(l.smem), st, maps, a);
  if (r != BL_OK || sp.split == 1) return r;
  const int64_t rw = (N % 4 == 0 ? M * (N / 4) : M * N);
  const dim3 rg(unsigned(grid_for(rw, 256)));
  if (dq)
    return launch_pdl(tc_reduce_kernel<true>, rg, dim3(256), 0, st, static_cast<const int32_t*>(a.part), sp.split,
                      M, N, s, beta, bias, Y, static_cast<int32_t*>(nullptr));
  return launch_pdl(tc_reduce_kernel<false>, rg, dim3(256), 0, st, static_cast<const int32_t*>(a.part), sp.split,
                    M, N, static_cast<const float*>(nullptr), static_cast<const float*>(nullptr),
                    static_cast<const float*>(nullptr), static_cast<float*>(nullptr), acc);
}

// Packed weights -> int8 rows in the workspace, for tensor-core GEMMs with more
// than kTcDecodeMaxTilesM row tiles (decoding inside the GEMM would repeat for
// every row tile there).
bl_status unpack_rows(const uint8_t* Wp, int64_t N, int64_t K, int64_t ldp, int8_t* Wq, int64_t ldk,
                      cudaStream_t st) {
  if (ldk % 16 != 0 || ldk < K || ldp % 16 != 0 || !is_aligned(Wp, 16) || !is_aligned(Wq, 16)) return BL_ERR_ALIGNMENT;
  unpack5_rows_kernel<<<grid_for(N * (ldp / 16), kUnpackThreads, 4), kUnpackThreads, 0, st>>>(Wp, N, ldp, Wq, ldk);
  return launch_status();
}

// ---- decode GEMV launches -------------------------------------------------
// One problem of a GEMV launch: Y from float32 X, or acc from X_q.
struct GemvCall {
  const float* X;
  const int8_t* Xq;
  int64_t ldxq;
  const void* W;
  int64_t ldw, N, K;
  const float* beta;
  const float* bias;
  float eps;
  float* Y;
  int32_t* acc;
};

template <int M, int CH, bool F>
bl_status launch_gemv_inst(const GemvArgs& a, int grid, uint32_t smem, cudaStream_t st) {
  constexpr int kMinBlocks = 1;   // the table and the staged rows hold one CTA per SM: registers are free
  auto kern = gemv_pack5_kernel<M, CH, F, kMinBlocks>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kGemvMaxSmem)) != cudaSuccess)
    return BL_ERR_CUDA;
  // programmatic dependent launch: the kernel's prologue (and, with static
  // weights, its weight copies) may overlap the previous kernel on the stream;
  // it waits (griddepcontrol.wait) before touching X, Y or acc
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(kGemvThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a) == cudaSuccess ? launch_status() : BL_ERR_CUDA;
}

template <bool F>
bl_status launch_gemv_f(int M, int ch, const GemvArgs& a, int grid, uint32_t smem, cudaStream_t st) {
  switch (M * 8 + ch) {
    case 1 * 8 + 1: return launch_gemv_inst<1, 1, F>(a, grid, smem, st);
    case 1 * 8 + 2: return launch_gemv_inst<1, 2, F>(a, grid, smem, st);
    case 1 * 8 + 3: return launch_gemv_inst<1, 3, F>(a, grid, smem, st);
    case 1 * 8 + 4: return launch_gemv_inst<1, 4, F>(a, grid, smem, st);
    case 2 * 8 + 1: return launch_gemv_inst<2, 1, F>(a, grid, smem, st);
    case 2 * 8 + 2: return launch_gemv_inst<2, 2, F>(a, grid, smem, st);
    case 3 * 8 + 1: return launch_gemv_inst<3, 1, F>(a, grid, smem, st);
    case 4 * 8 + 1: return launch_gemv_inst<4, 1, F>(a, grid, smem, st);
  }
  return BL_ERR_UNSUPPORTED;
}

// Up to kGemvMaxProbs problems with the same M in one launch; every call
// either quantizes float32 X (fused) or reads given X_q (not fused).
// CTAs of one GEMV launch per problem.  A CTA's time is modelled as a part
// that grows with K (every CTA copies and quantizes the whole X row: about as
// long as decoding four packed bytes per activation; one byte when the codes
// are given) plus its share of the packed bytes; the split evens out those
// times (water-filling: T with sum_i B_i / (T - r_i) = kGemvCtas, r_i the K
// part, B_i the packed bytes), rounded to whole CTAs, at least one per problem
// and at most one per row.
void gemv_split_ctas(const GemvCall* c, int n, bool fused, int64_t* want) {
  double r[kGemvMaxProbs], B[kGemvMaxProbs], rmax = 0.0, btot = 0.0;
  for (int i = 0; i < n; ++i) {
    r[i] = double(c[i].K) * (fused ? 4.0 : 1.0);
    B[i] = double(c[i].N) * double(c[i].ldw);
    rmax = r[i] > rmax ? r[i] : rmax;
    btot += B[i];
  }
  if (n == 1) {
    want[0] = std::min<int64_t>(kGemvCtas, c[0].N);
    return;
  }
  double lo = rmax, hi = rmax + btot;   // sum_i B_i / (T - r_i) falls from +inf to <= 1 over (lo, hi]
  for (int it = 0; it < 100; ++it) {
    const double T = 0.5 * (lo + hi);
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += B[i] / (T - r[i]);
    (s > double(kGemvCtas) ? lo : hi) = T;
  }
  double frac[kGemvMaxProbs];
  int64_t used = 0;
  for (int i = 0; i < n; ++i) {
    const double x = B[i] / (hi - r[i]);
    want[i] = std::max<int64_t>(1, int64_t(x));
    frac[i] = x - double(want[i]);
    used += want[i];
  }
  while (used < kGemvCtas) {   // the remainder to the largest fractions
    int best = -1;
    for (int i = 0; i < n; ++i)
      if (want[i] < c[i].N && (best < 0 || frac[i] > frac[best])) best = i;
    if (best < 0) break;
    ++want[best];
    frac[best] -= 1.0;
    ++used;
  }
  for (int i = 0; i < n; ++i) want[i] = std::min<int64_t>(want[i], c[i].N);
}

bl_status run_gemv_group(int64_t M, const GemvCall* c, int n, bool prefetch, cudaStream_t st) {
  if (n < 1 || n > kGemvMaxProbs || M < 1 || M > kGemvMaxM) return BL_ERR_UNSUPPORTED;
  const bool fused = c[0].X != nullptr;
  int ch = 1;
  for (int i = 0; i < n; ++i) {
    if ((c[i].X != nullptr) != fused) return BL_ERR_UNSUPPORTED;
    const int chi = gemv_chunks_per_lane(M, c[i].ldw);
    if (chi == 0) return BL_ERR_UNSUPPORTED;
    ch = chi > ch ? chi : ch;
  }
  GemvArgs a = {};
  a.nprob = n;
  (void)prefetch;   // the GEMV copies X before its weights either way
  int64_t wants[kGemvMaxProbs];
  gemv_split_ctas(c, n, fused, wants);
  int cta = 0;
  uint32_t smem = 0;
  for (int i = 0; i < n; ++i) {
    const int64_t want = wants[i];
    GemvProb& P = a.p[i];
    if (!gemv_plan_prob(M, c[i].N, c[i].K, c[i].ldw, int(want), ch, P)) return BL_ERR_UNSUPPORTED;
    P.X = c[i].X;
    P.Xq = c[i].Xq;
    P.ldxq = c[i].ldxq;
    P.Wp = static_cast<const uint8_t*>(c[i].W);
    P.N = c[i].N;
    P.K = c[i].K;
    P.ldp = c[i].ldw;
    P.beta = c[i].beta;
    P.bias = c[i].bias;
    P.eps = c[i].eps;
    P.Y = c[i].Y;
    P.acc = c[i].acc;
    if (!c[i].X || !is_aligned(c[i].X, 16)) P.xs_bytes = 0u;   // X read from global memory instead
    P.cta0 = cta;
    cta += int(ceil_div(c[i].N, int64_t(P.rows_per_cta)));   // every CTA has at least one row
    smem = P.smem > smem ? P.smem : smem;
  }
  return fused ? launch_gemv_f<true>(int(M), ch, a, cta, smem, st)
               : launch_gemv_f<false>(int(M), ch, a, cta, smem, st);
}

// The packed-trit GEMV for one call: Y from float32 X (fused quantization) or acc from X_q.
bl_status run_gemv(const float* X, const int8_t* Xq, int64_t ldxq, int64_t M, int64_t K,
                   const void* W, int64_t ldw, int64_t N, const float* beta, const float* bias,
                   float eps, float* Y, int32_t* acc, bool prefetch, cudaStream_t st) {
  GemvCall c = {X, Xq, ldxq, W, ldw, N, K, beta, bias, eps, Y, acc};
  return run_gemv_group(M, &c, 1, prefetch, st);
}

bl_status run_simt(const int8_t* Xq, int64_t ldx, int64_t M, int64_t K, const void* W,
                   bl_wfmt f, int64_t ldw, int64_t N, const float* s, const float* beta,
                   const float* bias, float* Y, int32_t* acc, cudaStream_t st) {
  const dim3 grid(unsigned(ceil_div(N, kSimtBN)), unsigned(ceil_div(M, kSimtBM)));
  if (grid.y > 65535u) return BL_ERR_UNSUPPORTED;
  const bool packed = f == BL_W_PACK5;
  if (Y) {
    if (packed) linear_simt_kernel<true, true><<<grid, 256, 0, st>>>(Xq, ldx, M, K, W, ldw, N, s, beta, bias, Y, nullptr);
    else linear_simt_kernel<false, true><<<grid, 256, 0, st>>>(Xq, ldx, M, K, W, ldw, N, s, beta, bias, Y, nullptr);
  } else {
    if (packed) linear_simt_kernel<true, false><<<grid, 256, 0, st>>>(Xq, ldx, M, K, W, ldw, N, nullptr, nullptr, nullptr, nullptr, acc);
    else linear_simt_kernel<false, false><<<grid, 256, 0, st>>>(Xq, ldx, M, K, W, ldw, N, nullptr, nullptr, nullptr, nullptr, acc);
  }
  return launch_status();
}

// ---- scratch for bl_linear_noalloc -------------------------------------------
// A file-scope device array: every GPU that loads the library holds it until the
// process exits.  Its name in host code is only a host-side stand-in, so the
// device address is looked up once per device with cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[BL_LINEAR_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (nullptr on error).
void* noalloc_scratch_ptr() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) return nullptr;
    g_noalloc_ptr[dev] = p;
  }
  return g_noalloc_ptr[dev];
}

}  // namespace
}  // namespace bl

using namespace bl;

extern "C" {

int64_t bl_pack5_ldp(int64_t K) { return K < 1 ? 0 : round_up(ceil_div(K, 5), 16); }

size_t bl_quantize_weights_workspace_size(int64_t N, int64_t K) {
  if (N < 1 || K < 1) return 0;
  return fused_shape(N, K) ? fused_ws_bytes(N, K, 0) : kAbsWsBytes;
}

bl_status bl_absmean(const float* W, int64_t N, int64_t K, float eps, float* beta_dev, void* ws,
                     size_t ws_bytes, cudaStream_t stream) {
  bl_status st = check_weights_args(W, N, K, beta_dev);
  if (st != BL_OK) return st;
  if (!eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if (!is_aligned(beta_dev, 4)) return BL_ERR_ALIGNMENT;
  if ((st = check_ws(ws, ws_bytes, kAbsWsBytes)) != BL_OK) return st;
  return launch_absmean(W, N * K, eps, beta_dev, ws, stream);
}

bl_status bl_ternarize(const float* W, int64_t N, int64_t K, const float* beta_dev, int8_t* Wq,
                       cudaStream_t stream) {
  bl_status st = check_weights_args(W, N, K, Wq);
  if (st != BL_OK) return st;
  if (!beta_dev) return BL_ERR_INVALID_ARG;
  if (!is_aligned(beta_dev, 4)) return BL_ERR_ALIGNMENT;
  const int64_t n = N * K;
  ternarize_i8_kernel<<<grid_for(ceil_div(n, 4), 256), 256, 0, stream>>>(W, n, beta_dev, Wq);
  return launch_status();
}

bl_status bl_ternarize_pack5(const float* W, int64_t N, int64_t K, const float* beta_dev,
                             uint8_t* Wp, int64_t ldp, cudaStream_t stream) {
  bl_status st = check_weights_args(W, N, K, Wp);
  if (st != BL_OK) return st;
  if (!beta_dev || ldp < ceil_div(K, 5)) return BL_ERR_INVALID_ARG;
  if (ldp % 16 != 0 || !is_aligned(Wp, 16) || !is_aligned(beta_dev, 4)) return BL_ERR_ALIGNMENT;
  ternarize_pack5_kernel<<<grid_for(N * (ldp / 4), 256), 256, 0, stream>>>(W, N, K, beta_dev, Wp, ldp);
  return launch_status();
}

bl_status bl_quantize_weights(const float* W, int64_t N, int64_t K, float eps, int8_t* Wq,
                              float* beta_dev, void* ws, size_t ws_bytes, cudaStream_t stream) {
  bl_status st = check_weights_args(W, N, K, Wq);
  if (st != BL_OK) return st;
  if (!eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if (!beta_dev) return BL_ERR_INVALID_ARG;
  if (!is_aligned(beta_dev, 4)) return BL_ERR_ALIGNMENT;
  if ((st = check_ws(ws, ws_bytes, kAbsWsBytes)) != BL_OK) return st;
  if (fused_shape(N, K) && is_aligned(W, 16) && is_aligned(Wq, 4) && ws_bytes >= fused_ws_bytes(N, K, 0)) {
    st = launch_wquant_fused(W, N, K, eps, Wq, K, false, beta_dev, ws, stream);
    if (st != BL_ERR_UNSUPPORTED) return st;
  }
  st = bl_absmean(W, N, K, eps, beta_dev, ws, ws_bytes, stream);
  if (st != BL_OK) return st;
  return bl_ternarize(W, N, K, beta_dev, Wq, stream);
}

bl_status bl_quantize_weights_pack5(const float* W, int64_t N, int64_t K, float eps,
                                    uint8_t* Wp, int64_t ldp, float* beta_dev, void* ws,
                                    size_t ws_bytes, cudaStream_t stream) {
  bl_status st = check_weights_args(W, N, K, Wp);
  if (st != BL_OK) return st;
  if (ldp < ceil_div(K, 5)) return BL_ERR_INVALID_ARG;
  if (ldp % 16 != 0 || !is_aligned(Wp, 16)) return BL_ERR_ALIGNMENT;
  if (!eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if (!beta_dev) return BL_ERR_INVALID_ARG;
  if (!is_aligned(beta_dev, 4)) return BL_ERR_ALIGNMENT;
  if ((st = check_ws(ws, ws_bytes, kAbsWsBytes)) != BL_OK) return st;
  if (fused_shape(N, K) && is_aligned(W, 16) && ws_bytes >= fused_ws_bytes(N, K, 0)) {
    st = launch_wquant_fused(W, N, K, eps, Wp, ldp, true, beta_dev, ws, stream);
    if (st != BL_ERR_UNSUPPORTED) return st;
  }
  st = bl_absmean(W, N, K, eps, beta_dev, ws, ws_bytes, stream);
  if (st != BL_OK) return st;
  return bl_ternarize_pack5(W, N, K, beta_dev, Wp, ldp, stream);
}

size_t bl_bitlinear_forward_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f) {
  if (M < 1 || N < 1 || K < 1 || (f != BL_W_I8 && f != BL_W_PACK5)) return 0;
  const size_t two = align_up(bl_quantize_weights_workspace_size(N, K)) + bl_linear_workspace_size(M, N, K, f);
  size_t one = 0;
  if (M <= kFwdMaxM && fused_shape(N, K) && N < (int64_t(1) << 31) && uint64_t(M * K * 4) <= kFwdXBytesMax)
    one = fused_ws_bytes(N, K, M);
  return align_up(two > one ? two : one);
}

bl_status bl_bitlinear_forward(const float* X, int64_t M, int64_t K, const float* W, bl_wfmt f,
                               int64_t N, float eps, void* Wout, int64_t ldo, float* beta_dev,
                               const float* bias, float* Y, void* ws, size_t ws_bytes,
                               cudaStream_t stream) {
  bl_status st = check_weights_args(W, N, K, Wout);
  if (st != BL_OK) return st;
  if (!X || !Y || !beta_dev || M < 1 || !eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if ((st = check_shape(M, K, N)) != BL_OK) return st;
  if (f == BL_W_PACK5) {
    if (ldo < ceil_div(K, 5)) return BL_ERR_INVALID_ARG;
    if (ldo % 16 != 0 || !is_aligned(Wout, 16)) return BL_ERR_ALIGNMENT;
  } else if (f == BL_W_I8) {
    if (ldo != K) return BL_ERR_INVALID_ARG;
  } else {
    return BL_ERR_INVALID_ARG;
  }
  if (!is_aligned(beta_dev, 4) || !is_aligned(X, 4) || !is_aligned(Y, 4)) return BL_ERR_ALIGNMENT;
  if ((st = check_ws(ws, ws_bytes, bl_bitlinear_forward_workspace_size(M, N, K, f))) != BL_OK) return st;
  if (fused_forward_ok(M, N, K, X, W) && (f == BL_W_PACK5 || is_aligned(Wout, 4))) {
    st = launch_wquant_fused(W, N, K, eps, Wout, ldo, f == BL_W_PACK5, beta_dev, ws, stream, M, X, bias, Y);
    if (st != BL_ERR_UNSUPPORTED) return st;
  }
  // otherwise the two calls: weight quantization, then the linear
  const size_t q = align_up(bl_quantize_weights_workspace_size(N, K));
  st = f == BL_W_PACK5
           ? bl_quantize_weights_pack5(W, N, K, eps, static_cast<uint8_t*>(Wout), ldo, beta_dev, ws, q, stream)
           : bl_quantize_weights(W, N, K, eps, static_cast<int8_t*>(Wout), beta_dev, ws, q, stream);
  if (st != BL_OK) return st;
  return bl_linear(X, M, K, Wout, f, N, ldo, beta_dev, bias, eps, Y, static_cast<char*>(ws) + q,
                   ws_bytes - q, stream);
}

bl_status bl_pack(const int8_t* Wq, int64_t N, int64_t K, uint8_t* Wp, int64_t ldp,
                  cudaStream_t stream) {
  if (!Wq || !Wp || N < 1 || K < 1 || ldp < ceil_div(K, 5)) return BL_ERR_INVALID_ARG;
  if (ldp % 16 != 0 || !is_aligned(Wp, 16)) return BL_ERR_ALIGNMENT;
  pack5_kernel<<<grid_for(N * (ldp / 4), 256), 256, 0, stream>>>(Wq, N, K, Wp, ldp);
  return launch_status();
}

bl_status bl_unpack(const uint8_t* Wp, int64_t N, int64_t K, int64_t ldp, int8_t* Wq,
                    cudaStream_t stream) {
  if (!Wq || !Wp || N < 1 || K < 1 || ldp < ceil_div(K, 5)) return BL_ERR_INVALID_ARG;
  unpack5_kernel<<<grid_for(N * ceil_div(K, 5), 256), 256, 0, stream>>>(Wp, N, K, ldp, Wq, K);
  return launch_status();
}

bl_status bl_quantize_act(const float* X, int64_t M, int64_t K, float eps, int8_t* Xq,
                          float* s, cudaStream_t stream) {
  if (M < 0 || K < 1 || !eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!X || !Xq || !s || M > (int64_t(1) << 31) - 1) return BL_ERR_INVALID_ARG;
  if (!is_aligned(X, 4) || !is_aligned(s, 4)) return BL_ERR_ALIGNMENT;
  launch_act_quant(X, M, K, eps, Xq, K, s, stream);
  return launch_status();
}

bl_status bl_rmsnorm_quantize_act(const float* X, int64_t M, int64_t K, const float* g, float eps_norm, float eps,
                                  int8_t* Xq, float* s, cudaStream_t stream) {
  if (M < 0 || K < 1 || K > kRnMaxK || !eps_ok(eps) || !eps_ok(eps_norm)) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!X || !g || !Xq || !s || M > (int64_t(1) << 31) - 1) return BL_ERR_INVALID_ARG;
  if (!is_aligned(X, 4) || !is_aligned(g, 4) || !is_aligned(s, 4)) return BL_ERR_ALIGNMENT;
  const int smem = int(K * 4);
  if (cudaFuncSetAttribute(rmsnorm_quant_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return BL_ERR_CUDA;
  rmsnorm_quant_kernel<<<unsigned(M), kRnThreads, smem, stream>>>(X, K, g, eps_norm, eps, Xq, K, s);
  return launch_status();
}

size_t bl_linear_ex_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path) {
  if (M < 0 || K < 1 || N < 1) return 0;
  path &= kPathMask;
  const int p = resolve_path(M, N, K, f, path, nullptr);
  if (p == BL_PATH_GEMV) return 0;   // activation quantization inside the GEMV: no scratch
  return lin_layout(M, K, N, p == BL_PATH_TC && tc_unpack(M, f), p == BL_PATH_TC ? tc_split(M, N, K, f).bytes : 0,
                    p == BL_PATH_TC && tc_swap(M, f))
      .total;
}

// bl_linear's workspace without the tensor-core K split's partials.
static size_t linear_ws_nosplit(int64_t M, int64_t N, int64_t K, bl_wfmt f) {
  const int p = resolve_path(M, N, K, f, BL_PATH_AUTO, nullptr);
  if (p == BL_PATH_GEMV) return 0;
  return lin_layout(M, K, N, p == BL_PATH_TC && tc_unpack(M, f), 0, p == BL_PATH_TC && tc_swap(M, f)).total;
}

size_t bl_linear_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f) {
  return bl_linear_ex_workspace_size(M, N, K, f, BL_PATH_AUTO);
}

// The argument checks of bl_linear (M == 0 passes once the rest is valid).
static bl_status check_linear(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f, int64_t N,
                              int64_t ldw, const float* beta_dev, const float* bias, float eps, const float* Y) {
  bl_status st = check_shape(M, K, N);
  if (st != BL_OK) return st;
  if (!eps_ok(eps)) return BL_ERR_INVALID_ARG;
  st = check_w(W, f, K, ldw);
  if (st != BL_OK || M == 0) return st;
  if (!X || !Y || !beta_dev) return BL_ERR_INVALID_ARG;
  if (!is_aligned(X, 4) || !is_aligned(Y, 4) || (bias && !is_aligned(bias, 4))) return BL_ERR_ALIGNMENT;
  return BL_OK;
}

// allow_split = false: the tensor-core GEMM runs without a K split (no partials
// in the workspace), for bl_linear_noalloc when the split would not fit.
static bl_status linear_impl(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f, int64_t N,
                             int64_t ldw, const float* beta_dev, const float* bias, float eps, float* Y,
                             void* ws, size_t ws_bytes, int path, bool allow_split, cudaStream_t stream) {
  const bool static_w = (path & BL_FLAG_STATIC_WEIGHTS) != 0;
  if (path & ~(kPathMask | BL_FLAG_STATIC_WEIGHTS)) return BL_ERR_INVALID_ARG;
  path &= kPathMask;
  if (path < BL_PATH_AUTO || path > BL_PATH_TC) return BL_ERR_INVALID_ARG;
  bl_status st = check_linear(X, M, K, W, f, N, ldw, beta_dev, bias, eps, Y);
  if (st != BL_OK || M == 0) return st;
  const int p = resolve_path(M, N, K, f, path, nullptr, true, ldw, W);
  if (p < 0) return BL_ERR_UNSUPPORTED;
  if (p == BL_PATH_GEMV)   // needs no workspace
    return run_gemv(X, nullptr, 0, M, K, W, ldw, N, beta_dev, bias, eps, Y, nullptr, static_w, stream);
  const size_t tcb = (p == BL_PATH_TC && allow_split) ? tc_split(M, N, K, f).bytes : 0;
  const bool swap = p == BL_PATH_TC && tc_swap(M, f);
  const LinWs l = lin_layout(M, K, N, p == BL_PATH_TC && tc_unpack(M, f), tcb, swap);
  if (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < l.total) return BL_ERR_WORKSPACE;
  void* tcws = tcb ? static_cast<char*>(ws) + l.tc_off : nullptr;   // null: no K split
  int8_t* Xq = reinterpret_cast<int8_t*>(static_cast<char*>(ws) + l.xq_off);
  float* s = reinterpret_cast<float*>(static_cast<char*>(ws) + l.s_off);
  if (swap)   // codes in the swapped GEMM's decode order
    launch_act_quant_dorder(X, M, K, eps, Xq, l.ldx, s, stream);
  else
    launch_act_quant(X, M, K, eps, Xq, l.ldx, s, stream);
  st = launch_status();
  if (st != BL_OK) return st;
  if (p == BL_PATH_TC) {
    if (tc_unpack(M, f)) {
      int8_t* scratch = reinterpret_cast<int8_t*>(static_cast<char*>(ws) + l.wq_off);
      st = unpack_rows(static_cast<const uint8_t*>(W), N, K, ldw, scratch, l.ldk, stream);
      if (st != BL_OK) return st;
      return run_tc(Xq, l.ldx, M, K, scratch, l.ldk, false, N, s, beta_dev, bias, Y, nullptr, tcws, tcb, stream);
    }
    if (swap)
      return run_swap(Xq, l.ldx, M, K, W, ldw, N, s, beta_dev, bias, Y, nullptr, tcws, tcb, static_w, stream);
    return run_tc(Xq, l.ldx, M, K, W, ldw, f == BL_W_PACK5, N, s, beta_dev, bias, Y, nullptr, tcws, tcb, stream);
  }
  return run_simt(Xq, l.ldx, M, K, W, f, ldw, N, s, beta_dev, bias, Y, nullptr, stream);
}

bl_status bl_linear_ex(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f,
                       int64_t N, int64_t ldw, const float* beta_dev, const float* bias,
                       float eps, float* Y, void* ws, size_t ws_bytes, int path,
                       cudaStream_t stream) {
  return linear_impl(X, M, K, W, f, N, ldw, beta_dev, bias, eps, Y, ws, ws_bytes, path, true, stream);
}

int bl_linear_plan(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path, int* launches) {
  path &= kPathMask;
  if (check_shape(M, K, N) != BL_OK || (f != BL_W_I8 && f != BL_W_PACK5)) return -1;
  if (path < BL_PATH_AUTO || path > BL_PATH_TC) return -1;
  return resolve_path(M, N, K, f, path, launches);
}

bl_status bl_linear(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f, int64_t N,
                    int64_t ldw, const float* beta_dev, const float* bias, float eps, float* Y,
                    void* ws, size_t ws_bytes, cudaStream_t stream) {
  return bl_linear_ex(X, M, K, W, f, N, ldw, beta_dev, bias, eps, Y, ws, ws_bytes,
                      BL_PATH_AUTO, stream);
}

// Whether a call of a group takes the decode GEMV (and so needs no workspace).
static bool group_gemv(const bl_linear_call& c) {
  return c.M >= 1 && resolve_path(c.M, c.N, c.K, c.f, BL_PATH_AUTO, nullptr, true, c.ldw, c.W) == BL_PATH_GEMV;
}

size_t bl_linear_group_workspace_size(const bl_linear_call* calls, int count) {
  if (!calls || count < 1) return 0;
  size_t t = 0;
  for (int i = 0; i < count; ++i)
    if (calls[i].M > 0 && !group_gemv(calls[i])) t += align_up(bl_linear_workspace_size(calls[i].M, calls[i].N, calls[i].K, calls[i].f));
  return t;
}

bl_status bl_linear_group(const bl_linear_call* calls, int count, int flags, void* ws, size_t ws_bytes,
                          cudaStream_t stream) {
  if (count < 0 || (count > 0 && !calls)) return BL_ERR_INVALID_ARG;
  if (flags & ~BL_FLAG_STATIC_WEIGHTS) return BL_ERR_INVALID_ARG;
  // every call is checked before anything is launched
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    const bl_status st = check_linear(c.X, c.M, c.K, c.W, c.f, c.N, c.ldw, c.beta_dev, c.bias, c.eps, c.Y);
    if (st != BL_OK) return st;
  }
  const size_t need = bl_linear_group_workspace_size(calls, count);
  if (need && (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < need)) return BL_ERR_WORKSPACE;
  // decode-GEMV calls: one launch per M, up to kGemvMaxProbs problems each
  for (int64_t m = 1; m <= kGemvMaxM; ++m) {
    GemvCall g[kGemvMaxProbs];
    int n = 0;
    for (int i = 0; i <= count; ++i) {
      if (i < count && calls[i].M == m && group_gemv(calls[i])) {
        const bl_linear_call& c = calls[i];
        g[n++] = GemvCall{c.X, nullptr, 0, c.W, c.ldw, c.N, c.K, c.beta_dev, c.bias, c.eps, c.Y, nullptr};
      }
      if (n == kGemvMaxProbs || (i == count && n > 0)) {
        const bl_status st = run_gemv_group(m, g, n, (flags & BL_FLAG_STATIC_WEIGHTS) != 0, stream);
        if (st != BL_OK) return st;
        n = 0;
      }
    }
  }
  // the rest, each as bl_linear with its own part of the workspace
  size_t off = 0;
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    if (c.M == 0 || group_gemv(c)) continue;
    const size_t wsz = bl_linear_workspace_size(c.M, c.N, c.K, c.f);
    const bl_status st = linear_impl(c.X, c.M, c.K, c.W, c.f, c.N, c.ldw, c.beta_dev, c.bias, c.eps, c.Y,
                                     static_cast<char*>(ws) + off, wsz, BL_PATH_AUTO | flags, true, stream);
    if (st != BL_OK) return st;
    off += align_up(wsz);
  }
  return BL_OK;
}

// One copy of bl_linear_group_host: `bytes` from src to dst.
struct CopySpan {
  char* dst;
  const char* src;
  size_t bytes;
};

// Enqueues the spans in order, one cudaMemcpyAsync per run of spans that follow
// one another end to end on both sides (empty spans are skipped).
static bl_status enqueue_copy_runs(const std::vector<CopySpan>& s, cudaMemcpyKind kind, cudaStream_t stream) {
  size_t i = 0;
  while (i < s.size()) {
    if (s[i].bytes == 0) {
      ++i;
      continue;
    }
    CopySpan run = s[i];
    size_t j = i + 1;
    for (; j < s.size(); ++j) {
      if (s[j].bytes == 0) continue;
      if (s[j].dst != run.dst + run.bytes || s[j].src != run.src + run.bytes) break;
      run.bytes += s[j].bytes;
    }
    if (cudaMemcpyAsync(run.dst, run.src, run.bytes, kind, stream) != cudaSuccess) return BL_ERR_CUDA;
    i = j;
  }
  return BL_OK;
}

// The device address through which kernels reach host memory at p (page-locked
// and mapped into the device's address space), else nullptr (pageable memory,
// device memory, or an unknown pointer).
static void* host_alias(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

// Mapped host rows moved by span_copy_kernel rather than the copy engine, up to
// this many bytes per call (beyond it the copy engine's bandwidth wins).
constexpr size_t kSpanKernelMaxBytes = size_t(4) << 20;

// Copies the runs of `s` (host-mapped sources, device destinations) with
// span_copy_kernel, kSpanMax spans per launch, programmatic dependent launch.
static bl_status enqueue_span_kernels(const std::vector<CopySpan>& s, cudaStream_t stream) {
  std::vector<CopySpan> runs;
  for (const CopySpan& c : s) {
    if (c.bytes == 0) continue;
    if (!runs.empty() && runs.back().dst + runs.back().bytes == c.dst && runs.back().src + runs.back().bytes == c.src)
      runs.back().bytes += c.bytes;
    else
      runs.push_back(c);
  }
  for (size_t i0 = 0; i0 < runs.size(); i0 += kSpanMax) {
    const int n = int(std::min(runs.size() - i0, size_t(kSpanMax)));
    bool v16 = true;
    for (int j = 0; j < n; ++j) {
      const CopySpan& c = runs[i0 + j];
      v16 = v16 && is_aligned(c.dst, 16) && is_aligned(c.src, 16) && c.bytes % 16 == 0;
    }
    const int unit = v16 ? 16 : 4;
    SpanCopy a = {};
    a.n = n;
    a.first[0] = 0;
    for (int j = 0; j < n; ++j) {
      a.dst[j] = runs[i0 + j].dst;
      a.src[j] = runs[i0 + j].src;
      a.first[j + 1] = a.first[j] + int64_t(runs[i0 + j].bytes / unit);
    }
    for (int j = n; j < kSpanMax; ++j) a.first[j + 1] = a.first[n];
    const int64_t blocks = std::min<int64_t>(ceil_div(a.first[n], int64_t(kSpanThreads) * kSpanPre), 8 * 148);
    const bl_status st = v16 ? launch_pdl(span_copy_kernel<16>, dim3(unsigned(blocks)), dim3(kSpanThreads), 0, stream, a)
                             : launch_pdl(span_copy_kernel<4>, dim3(unsigned(blocks)), dim3(kSpanThreads), 0, stream, a);
    if (st != BL_OK) return st;
  }
  return BL_OK;
}

bl_status bl_linear_group_host(const bl_linear_call* calls, const bl_host_io* io, int count, int flags,
                               void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (count < 0 || (count > 0 && (!calls || !io))) return BL_ERR_INVALID_ARG;
  if (flags & ~BL_FLAG_STATIC_WEIGHTS) return BL_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    const bl_status st = check_linear(c.X, c.M, c.K, c.W, c.f, c.N, c.ldw, c.beta_dev, c.bias, c.eps, c.Y);
    if (st != BL_OK) return st;
    if (c.M > 0 && (!io[i].X_host || !io[i].Y_host)) return BL_ERR_INVALID_ARG;
  }
  const size_t need = bl_linear_group_workspace_size(calls, count);
  if (need && (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < need)) return BL_ERR_WORKSPACE;
  // inputs: mapped host rows by span_copy_kernel (up to kSpanKernelMaxBytes),
  // the rest by the copy engine; results: a decode-GEMV call whose Y_host is
  // mapped gets it as its Y (plain stores over the bus), the rest are copied back
  std::vector<bl_linear_call> run(calls, calls + count);
  std::vector<CopySpan> in_k, in_c, out_c;
  size_t kbytes = 0;
  for (int i = 0; i < count; ++i) {
    const bl_linear_call& c = calls[i];
    if (c.M == 0) continue;
    char* xd = reinterpret_cast<char*>(const_cast<float*>(c.X));
    const size_t xb = size_t(c.M) * size_t(c.K) * 4, yb = size_t(c.M) * size_t(c.N) * 4;
    const void* xa = host_alias(io[i].X_host);
    if (xa && kbytes + xb <= kSpanKernelMaxBytes) {
      in_k.push_back(CopySpan{xd, static_cast<const char*>(xa), xb});
      kbytes += xb;
    } else {
      in_c.push_back(CopySpan{xd, reinterpret_cast<const char*>(io[i].X_host), xb});
    }
    void* ya = group_gemv(c) ? host_alias(io[i].Y_host) : nullptr;
    if (ya)
      run[size_t(i)].Y = static_cast<float*>(ya);
    else
      out_c.push_back(CopySpan{reinterpret_cast<char*>(io[i].Y_host), reinterpret_cast<const char*>(c.Y), yb});
  }
  bl_status st = enqueue_copy_runs(in_c, cudaMemcpyHostToDevice, stream);
  if (st == BL_OK) st = enqueue_span_kernels(in_k, stream);
  if (st == BL_OK) st = bl_linear_group(run.data(), count, flags, ws, ws_bytes, stream);
  if (st == BL_OK) st = enqueue_copy_runs(out_c, cudaMemcpyDeviceToHost, stream);
  return st;
}

bl_status bl_linear_noalloc(const float* X, int64_t M, int64_t K, const void* W, bl_wfmt f,
                            int64_t N, int64_t ldw, const float* beta_dev, const float* bias,
                            float eps, float* Y, cudaStream_t stream) {
  bl_status st = check_shape(M, K, N);
  if (st != BL_OK) return st;
  if (!eps_ok(eps)) return BL_ERR_INVALID_ARG;
  if ((st = check_w(W, f, K, ldw)) != BL_OK) return st;
  if (M == 0) return BL_OK;
  // the tensor-core K split only if its partials fit the array as well
  const bool split = bl_linear_workspace_size(M, N, K, f) <= BL_LINEAR_NOALLOC_SCRATCH_BYTES;
  if (!split && linear_ws_nosplit(M, N, K, f) > BL_LINEAR_NOALLOC_SCRATCH_BYTES) return BL_ERR_WORKSPACE;
  void* scratch = noalloc_scratch_ptr();
  if (!scratch) return BL_ERR_CUDA;
  return linear_impl(X, M, K, W, f, N, ldw, beta_dev, bias, eps, Y, scratch, BL_LINEAR_NOALLOC_SCRATCH_BYTES,
                     BL_PATH_AUTO, split, stream);
}

size_t bl_linear_acc_workspace_size(int64_t M, int64_t N, int64_t K, bl_wfmt f, int path) {
  if (M < 1 || N < 1 || K < 1) return 0;
  path &= kPathMask;
  const int p = resolve_path(M, N, K, f, path, nullptr, false);
  if (p != BL_PATH_TC) return 0;
  if (tc_swap(M, f))   // the split's partials, then the codes in decode order
    return tc_split(M, N, K, f).bytes + align_up(size_t(M) * size_t(swap_ldx(K)));
  return (tc_unpack(M, f) ? align_up(size_t(N) * size_t(round_up(K, 16))) : 0) + tc_split(M, N, K, f).bytes;
}

// no_ws: bl_linear_acc, which takes no workspace: packed weights are then
// decoded inside the un-swapped tensor-core GEMM at any M, and K is not split
// (the swapped GEMM needs the codes in decode order, a copy in the workspace).
static bl_status linear_acc_impl(const int8_t* Xq, int64_t M, int64_t K, const void* W, bl_wfmt f, int64_t N,
                          int64_t ldw, int32_t* acc, void* ws, size_t ws_bytes, int path, bool no_ws,
                          cudaStream_t stream) {
  const bool static_w = (path & BL_FLAG_STATIC_WEIGHTS) != 0;
  if (path & ~(kPathMask | BL_FLAG_STATIC_WEIGHTS)) return BL_ERR_INVALID_ARG;
  path &= kPathMask;
  bl_status st = check_shape(M, K, N);
  if (st != BL_OK) return st;
  st = check_w(W, f, K, ldw);
  if (st != BL_OK) return st;
  if (path < BL_PATH_AUTO || path > BL_PATH_TC) return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!Xq || !acc) return BL_ERR_INVALID_ARG;
  if (!is_aligned(acc, 4)) return BL_ERR_ALIGNMENT;
  int p = resolve_path(M, N, K, f, path, nullptr, false, ldw, W);
  const bool swap = p == BL_PATH_TC && tc_swap(M, f) && !no_ws;
  // X_q given by the caller: the un-swapped tensor-core GEMM needs a TMA-able
  // [M, K] int8 matrix (the swapped one reads a decode-order copy)
  const bool tc_x_ok = swap || (K % 16 == 0 && is_aligned(Xq, 16));
  if (p == BL_PATH_TC && !tc_x_ok) {
    if (path == BL_PATH_TC) return BL_ERR_UNSUPPORTED;
    p = resolve_path(M, N, K, f, BL_PATH_GEMV, nullptr, false) >= 0 ? BL_PATH_GEMV : BL_PATH_SIMT;
  }
  if (p < 0) return BL_ERR_UNSUPPORTED;
  if (p == BL_PATH_GEMV)
    return run_gemv(nullptr, Xq, K, M, K, W, ldw, N, nullptr, nullptr, 0.f, nullptr, acc, static_w, stream);
  if (p == BL_PATH_TC && swap) {
    const int64_t ldd = swap_ldx(K);
    const TcSplit sp = tc_split(M, N, K, f);
    const size_t need = sp.bytes + align_up(size_t(M) * size_t(ldd));
    if (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < need) return BL_ERR_WORKSPACE;
    int8_t* Xd = static_cast<int8_t*>(ws) + sp.bytes;
    bl_status st2 = launch_pdl(xq_dorder_kernel, dim3(unsigned(grid_for(M * (ldd / 4), 256))), dim3(256), 0,
                               stream, Xq, K, M, K, Xd, ldd);
    if (st2 != BL_OK) return st2;
    return run_swap(Xd, ldd, M, K, W, ldw, N, nullptr, nullptr, nullptr, nullptr, acc, sp.bytes ? ws : nullptr,
                    sp.bytes, static_w, stream);
  }
  if (p == BL_PATH_TC) {
    const bool unp = !no_ws && tc_unpack(M, f);
    const size_t wq = unp ? align_up(size_t(N) * size_t(round_up(K, 16))) : 0;
    const size_t need = no_ws ? 0 : wq + tc_split(M, N, K, f).bytes;
    if (need && (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < need)) return BL_ERR_WORKSPACE;
    void* tcws = need > wq ? static_cast<char*>(ws) + wq : nullptr;
    const size_t tcb = need > wq ? ws_bytes - wq : 0;
    if (unp) {
      int8_t* scratch = static_cast<int8_t*>(ws);
      bl_status st2 = unpack_rows(static_cast<const uint8_t*>(W), N, K, ldw, scratch, round_up(K, 16), stream);
      if (st2 != BL_OK) return st2;
      return run_tc(Xq, K, M, K, scratch, round_up(K, 16), false, N, nullptr, nullptr, nullptr, nullptr, acc,
                    tcws, tcb, stream);
    }
    return run_tc(Xq, K, M, K, W, ldw, f == BL_W_PACK5, N, nullptr, nullptr, nullptr, nullptr, acc, tcws, tcb,
                  stream);
  }
  return run_simt(Xq, K, M, K, W, f, ldw, N, nullptr, nullptr, nullptr, nullptr, acc, stream);
}

bl_status bl_linear_acc_ex(const int8_t* Xq, int64_t M, int64_t K, const void* W, bl_wfmt f,
                           int64_t N, int64_t ldw, int32_t* acc, void* ws, size_t ws_bytes,
                           int path, cudaStream_t stream) {
  return linear_acc_impl(Xq, M, K, W, f, N, ldw, acc, ws, ws_bytes, path, false, stream);
}

bl_status bl_linear_acc(const int8_t* Xq, int64_t M, int64_t K, const void* W, bl_wfmt f,
                        int64_t N, int64_t ldw, int32_t* acc, cudaStream_t stream) {
  return linear_acc_impl(Xq, M, K, W, f, N, ldw, acc, nullptr, 0, BL_PATH_AUTO, true, stream);
}

// ---- straight-through backward ---------------------------------------------------
struct BwLayout {
  int64_t ldN, ldM;
  size_t dx_a, dx_b, dw_a, dw_b, total;   // bytes of one hi (or lo) array of each operand
};
static BwLayout bw_layout(int64_t M, int64_t N, int64_t K) {
  BwLayout l;
  l.ldN = round_up(N, 4);
  l.ldM = round_up(M, 4);
  l.dx_a = align_up(size_t(M) * size_t(l.ldN) * 4);
  l.dx_b = align_up(size_t(K) * size_t(l.ldN) * 4);
  l.dw_a = align_up(size_t(N) * size_t(l.ldM) * 4);
  l.dw_b = align_up(size_t(K) * size_t(l.ldM) * 4);
  const size_t dx = 2 * (l.dx_a + l.dx_b), dw = 2 * (l.dw_a + l.dw_b);
  l.total = dx > dw ? dx : dw;
  return l;
}

size_t bl_linear_backward_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1) return 0;
  return bw_layout(M, N, K).total;
}

bl_status bl_linear_backward(const float* dY, const float* X, const float* W, int64_t M, int64_t N, int64_t K,
                             float* dX, float* dW, float* db, void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (M < 0 || N < 1 || K < 1 || M > (int64_t(1) << 31) - 1 || N > (int64_t(1) << 31) - 1 ||
      K > (int64_t(1) << 31) - 1)
    return BL_ERR_INVALID_ARG;
  if (M == 0) return BL_OK;
  if (!dY || (dX && !W) || (dW && !X)) return BL_ERR_INVALID_ARG;
  for (const void* p : {static_cast<const void*>(dY), static_cast<const void*>(X), static_cast<const void*>(W),
                        static_cast<const void*>(dX), static_cast<const void*>(dW), static_cast<const void*>(db)})
    if (p && !is_aligned(p, 4)) return BL_ERR_ALIGNMENT;
  const BwLayout l = bw_layout(M, N, K);
  if ((dX || dW) && (!ws || !is_aligned(ws, kWsAlign) || ws_bytes < l.total)) return BL_ERR_WORKSPACE;
  char* w = static_cast<char*>(ws);
  bl_status st = BL_OK;
  if (dX) {   // dX [M, K] = dY [M, N] W [N, K]: A = dY (K-major over n), B = W^T [K, N]
    float* ahi = reinterpret_cast<float*>(w);
    float* alo = reinterpret_cast<float*>(w + l.dx_a);
    float* bhi = reinterpret_cast<float*>(w + 2 * l.dx_a);
    float* blo = reinterpret_cast<float*>(w + 2 * l.dx_a + l.dx_b);
    split_tf32_kernel<false><<<grid_for(M * l.ldN, 256), 256, 0, stream>>>(dY, M, N, N, ahi, alo, l.ldN);
    split_tf32_kernel<true><<<grid_for(ceil_div(l.ldN, 32) * ceil_div(K, 32), 1), 256, 0, stream>>>(W, N, K, K, bhi,
                                                                                                   blo, l.ldN);
    if ((st = launch_status()) != BL_OK) return st;
    if ((st = run_tf32x3(ahi, alo, bhi, blo, l.ldN, M, K, N, dX, stream)) != BL_OK) return st;
  }
  if (dW) {   // dW [N, K] = dY^T [N, M] X [M, K]: A = dY^T [N, M], B = X^T [K, M]
    float* ahi = reinterpret_cast<float*>(w);
    float* alo = reinterpret_cast<float*>(w + l.dw_a);
    float* bhi = reinterpret_cast<float*>(w + 2 * l.dw_a);
    float* blo = reinterpret_cast<float*>(w + 2 * l.dw_a + l.dw_b);
    split_tf32_kernel<true><<<grid_for(ceil_div(l.ldM, 32) * ceil_div(N, 32), 1), 256, 0, stream>>>(dY, M, N, N, ahi,
                                                                                                   alo, l.ldM);
    split_tf32_kernel<true><<<grid_for(ceil_div(l.ldM, 32) * ceil_div(K, 32), 1), 256, 0, stream>>>(X, M, K, K, bhi,
                                                                                                   blo, l.ldM);
    if ((st = launch_status()) != BL_OK) return st;
    if ((st = run_tf32x3(ahi, alo, bhi, blo, l.ldM, N, K, M, dW, stream)) != BL_OK) return st;
  }
  if (db) {
    colsum_kernel<<<grid_for(N, 256), 256, 0, stream>>>(dY, M, N, db);
    if ((st = launch_status()) != BL_OK) return st;
  }
  return BL_OK;
}

// ---- deployed checkpoint ------------------------------------------------------
bl_status bl_save_deployed(const char* path, const bl_deployed_layer* layers, int count, cudaStream_t stream) {
  if (!path || count < 0 || (count > 0 && !layers)) return BL_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    const bl_deployed_layer& L = layers[i];
    if (L.N < 1 || L.K < 1 || L.K > kMaxK || L.N > (int64_t(1) << 40) || !L.Wp || !L.beta_dev) return BL_ERR_INVALID_ARG;
    if (L.ldp < ceil_div(L.K, 5)) return BL_ERR_INVALID_ARG;
    if (L.name && strlen(L.name) > io::kMaxName) return BL_ERR_INVALID_ARG;
  }
  if (count > 0 && cudaStreamSynchronize(stream) != cudaSuccess) return BL_ERR_CUDA;
  io::File file;
  file.f = fopen(path, "wb");
  if (!file.f) return BL_ERR_IO;
  bl_status st = BL_OK;
  unsigned char h[24];
  memcpy(h, io::kMagic, 4);
  io::put_u32(h + 4, io::kVersion);
  io::put_u32(h + 8, uint32_t(count));
  io::put_u32(h + 12, 0u);
  if (fwrite(h, 1, 16, file.f) != 16) st = BL_ERR_IO;
  unsigned char* buf = nullptr;
  for (int i = 0; i < count && st == BL_OK; ++i) {
    const bl_deployed_layer& L = layers[i];
    const uint32_t nlen = L.name ? uint32_t(strlen(L.name)) : 0u;
    uint32_t beta_bits = 0;
    if (cudaMemcpyAsync(&beta_bits, L.beta_dev, 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess) {
      st = BL_ERR_CUDA;
      break;
    }
    io::put_u32(h, nlen);
    if (fwrite(h, 1, 4, file.f) != 4 || (nlen && fwrite(L.name, 1, nlen, file.f) != nlen)) {
      st = BL_ERR_IO;
      break;
    }
    io::put_u64(h, uint64_t(L.N));
    io::put_u64(h + 8, uint64_t(L.K));
    io::put_u32(h + 16, L.bias_dev ? 1u : 0u);
    io::put_u32(h + 20, beta_bits);
    if (fwrite(h, 1, 24, file.f) != 24) {
      st = BL_ERR_IO;
      break;
    }
    const size_t cb = size_t(ceil_div(L.K, 5));
    const int64_t rows_per = int64_t(io::kIoChunk / cb) > 0 ? int64_t(io::kIoChunk / cb) : 1;
    if (!buf && !(buf = static_cast<unsigned char*>(malloc(io::kIoChunk > cb ? io::kIoChunk : cb)))) {
      st = BL_ERR_IO;
      break;
    }
    for (int64_t r0 = 0; r0 < L.N && st == BL_OK; r0 += rows_per) {
      const int64_t nr = L.N - r0 < rows_per ? L.N - r0 : rows_per;
      if (cudaMemcpy2DAsync(buf, cb, L.Wp + r0 * L.ldp, size_t(L.ldp), cb, size_t(nr), cudaMemcpyDeviceToHost,
                            stream) != cudaSuccess ||
          cudaStreamSynchronize(stream) != cudaSuccess)
        st = BL_ERR_CUDA;
      else if (fwrite(buf, 1, cb * size_t(nr), file.f) != cb * size_t(nr))
        st = BL_ERR_IO;
    }
    if (st == BL_OK && L.bias_dev) {
      const int64_t per = int64_t(io::kIoChunk / 4);
      for (int64_t n0 = 0; n0 < L.N && st == BL_OK; n0 += per) {
        const int64_t nn = L.N - n0 < per ? L.N - n0 : per;
        float* fb = reinterpret_cast<float*>(buf);
        if (cudaMemcpyAsync(fb, L.bias_dev + n0, size_t(nn) * 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess) {
          st = BL_ERR_CUDA;
          break;
        }
        for (int64_t j = 0; j < nn; ++j) {   // little-endian float32 bits
          uint32_t u;
          memcpy(&u, fb + j, 4);
          io::put_u32(buf + 4 * j, u);
        }
        if (fwrite(buf, 1, size_t(nn) * 4, file.f) != size_t(nn) * 4) st = BL_ERR_IO;
      }
    }
  }
  free(buf);
  if (fclose(file.f) != 0 && st == BL_OK) st = BL_ERR_IO;
  file.f = nullptr;
  if (st != BL_OK) remove(path);
  return st;
}

bl_status bl_deployed_count(const char* path, int* count) {
  if (!path || !count) return BL_ERR_INVALID_ARG;
  io::File file;
  const int n = io::open_checked(path, file);
  if (n < 0) return BL_ERR_IO;
  io::Record r;
  for (int i = 0; i < n; ++i)
    if (!io::read_record(file.f, r)) return BL_ERR_IO;
  const long end = ftell(file.f);
  if (fseek(file.f, 0, SEEK_END) != 0 || ftell(file.f) != end) return BL_ERR_IO;   // short or trailing bytes
  *count = n;
  return BL_OK;
}

bl_status bl_deployed_layer_info(const char* path, int index, int64_t* N, int64_t* K, int* has_bias, char* name,
                                 size_t name_cap) {
  if (!path || index < 0) return BL_ERR_INVALID_ARG;
  int n = 0;
  bl_status st = bl_deployed_count(path, &n);
  if (st != BL_OK) return st;
  if (index >= n) return BL_ERR_INVALID_ARG;
  io::File file;
  io::Record r;
  if (io::open_checked(path, file) < 0 || !io::seek_layer(file, index, r)) return BL_ERR_IO;
  if (N) *N = int64_t(r.N);
  if (K) *K = int64_t(r.K);
  if (has_bias) *has_bias = int(r.flags & 1u);
  if (name && name_cap) {
    strncpy(name, r.name, name_cap - 1);
    name[name_cap - 1] = '\0';
  }
  return BL_OK;
}

bl_status bl_load_deployed_layer(const char* path, int index, uint8_t* Wp, int64_t ldp, float* beta_dev,
                                 float* bias_dev, cudaStream_t stream) {
  if (!path || index < 0 || !Wp || !beta_dev) return BL_ERR_INVALID_ARG;
  int n = 0;
  bl_status st = bl_deployed_count(path, &n);
  if (st != BL_OK) return st;
  if (index >= n) return BL_ERR_INVALID_ARG;
  io::File file;
  io::Record r;
  if (io::open_checked(path, file) < 0 || !io::seek_layer(file, index, r)) return BL_ERR_IO;
  const int64_t N = int64_t(r.N), K = int64_t(r.K);
  const size_t cb = size_t(ceil_div(K, 5));
  if (ldp < int64_t(cb)) return BL_ERR_INVALID_ARG;
  if (ldp % 16 != 0 || !is_aligned(Wp, 16) || !is_aligned(beta_dev, 4)) return BL_ERR_ALIGNMENT;
  if (bias_dev && !(r.flags & 1u)) return BL_ERR_INVALID_ARG;
  if (fseek(file.f, r.packed_off, SEEK_SET) != 0) return BL_ERR_IO;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return BL_ERR_CUDA;
  const int64_t rows_per = int64_t(io::kIoChunk / cb) > 0 ? int64_t(io::kIoChunk / cb) : 1;
  unsigned char* buf = static_cast<unsigned char*>(malloc(io::kIoChunk > cb ? io::kIoChunk : cb));
  if (!buf) return BL_ERR_IO;
  for (int64_t r0 = 0; r0 < N && st == BL_OK; r0 += rows_per) {
    const int64_t nr = N - r0 < rows_per ? N - r0 : rows_per;
    const size_t nb = cb * size_t(nr);
    if (fread(buf, 1, nb, file.f) != nb) {
      st = BL_ERR_IO;
      break;
    }
    for (size_t j = 0; j < nb; ++j)
      if (buf[j] > 242) st = BL_ERR_IO;    // not a five-trit code
    if (st == BL_OK && (cudaMemcpy2DAsync(Wp + r0 * ldp, size_t(ldp), buf, cb, cb, size_t(nr), cudaMemcpyHostToDevice,
                                          stream) != cudaSuccess ||
                        cudaStreamSynchronize(stream) != cudaSuccess))
      st = BL_ERR_CUDA;
  }
  // whole padding bytes of every row: five zero trits each
  if (st == BL_OK && ldp > int64_t(cb) &&
      cudaMemset2DAsync(Wp + cb, size_t(ldp), 121, size_t(ldp) - cb, size_t(N), stream) != cudaSuccess)
    st = BL_ERR_CUDA;
  if (st == BL_OK) {
    float beta;
    memcpy(&beta, &r.beta_bits, 4);
    if (cudaMemcpyAsync(beta_dev, &beta, 4, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      st = BL_ERR_CUDA;
  }
  if (st == BL_OK && bias_dev) {
    const int64_t per = int64_t(io::kIoChunk / 4);
    for (int64_t n0 = 0; n0 < N && st == BL_OK; n0 += per) {
      const int64_t nn = N - n0 < per ? N - n0 : per;
      if (fread(buf, 1, size_t(nn) * 4, file.f) != size_t(nn) * 4) {
        st = BL_ERR_IO;
        break;
      }
      float* fb = reinterpret_cast<float*>(buf);
      for (int64_t j = 0; j < nn; ++j) {
        const uint32_t u = io::get_u32(buf + 4 * j);
        memcpy(fb + j, &u, 4);
      }
      if (cudaMemcpyAsync(bias_dev + n0, fb, size_t(nn) * 4, cudaMemcpyHostToDevice, stream) != cudaSuccess ||
          cudaStreamSynchronize(stream) != cudaSuccess)
        st = BL_ERR_CUDA;
    }
  }
  free(buf);
  return st;
}

// One thread waits on a phase that nothing completes, with a short limit.
__global__ void selftest_timeout_kernel(uint64_t limit_ns) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait(&bar, 0u, limit_ns)) raise_status(kDevTimeout);
}

bl_status bl_selftest_wait_timeout(int64_t limit_ns, cudaStream_t stream) {
  if (limit_ns < 1000 || limit_ns > int64_t(kWaitLimitNs)) return BL_ERR_INVALID_ARG;
  selftest_timeout_kernel<<<1, 1, 0, stream>>>(uint64_t(limit_ns));
  return launch_status();
}

bl_status bl_sync_status(cudaStream_t stream) {
  if (cudaStreamSynchronize(stream) != cudaSuccess) return BL_ERR_CUDA;
  unsigned int word = 0u, zero = 0u;
  if (cudaMemcpyFromSymbol(&word, g_status, sizeof(word)) != cudaSuccess) return BL_ERR_CUDA;
  if (word && cudaMemcpyToSymbol(g_status, &zero, sizeof(zero)) != cudaSuccess) return BL_ERR_CUDA;
  if (word & kDevTimeout) return BL_ERR_DEVICE_TIMEOUT;
  if (word & kDevBadWorkspace) return BL_ERR_WORKSPACE;
  if (word & kDevNonFinite) return BL_ERR_NONFINITE;
  return launch_status();
}

const char* bl_status_string(bl_status s) {
  switch (s) {
    case BL_OK: return "BL_OK";
    case BL_ERR_INVALID_ARG: return "BL_ERR_INVALID_ARG";
    case BL_ERR_ALIGNMENT: return "BL_ERR_ALIGNMENT";
    case BL_ERR_UNSUPPORTED: return "BL_ERR_UNSUPPORTED";
    case BL_ERR_WORKSPACE: return "BL_ERR_WORKSPACE";
    case BL_ERR_CUDA: return "BL_ERR_CUDA";
    case BL_ERR_DEVICE_TIMEOUT: return "BL_ERR_DEVICE_TIMEOUT";
    case BL_ERR_NONFINITE: return "BL_ERR_NONFINITE";
    case BL_ERR_IO: return "BL_ERR_IO";
  }
  return "BL_ERR_UNKNOWN";
}

}  // extern "C"
