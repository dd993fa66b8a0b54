// General-shape ternary x int8 contraction on the CUDA cores (dp4a).
//
// acc[m,n] = sum_k x_q[m,k] * W_q[n,k]: the integer product x_q W_q^T of the
// deployed-path equation y = (x_q W_q^T)(s beta) + b ("ultragraph -- when the
// graph is the 1-bit LLM, part 2", section "autograd on a byte-graph").  With
// trits the products are add / subtract / skip ("a 1-bit llm, from scratch",
// "the interesting bit"); dp4a does four of them per instruction, exactly.
//
// This kernel takes any M, N, K, either weight format and any alignment; the
// specialised GEMV and tensor-core kernels cover the shapes that matter for
// speed.  64x64 output tile per CTA, K staged 80 at a time (16 packed bytes).
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kSimtBM = 64, kSimtBN = 64, kSimtBK = 80, kSimtKW = kSimtBK / 4;

// Four int8 from row `r` of a byte matrix at column k (zero past K or past rows).
__device__ __forceinline__ uint32_t load_i8x4(const int8_t* base, int64_t ld, int64_t r,
                                              int64_t rows, int64_t k, int64_t K, bool vec) {
  if (r >= rows || k >= K) return 0u;
  const int8_t* p = base + r * ld + k;
  if (vec && k + 4 <= K) return *reinterpret_cast<const uint32_t*>(p);
  uint32_t w = 0u;
  for (int i = 0; i < 4 && k + i < K; ++i) w |= uint32_t(uint8_t(p[i])) << (8 * i);
  return w;
}

template <bool kPacked, bool kDequant>
__global__ void __launch_bounds__(256)
linear_simt_kernel(const int8_t* __restrict__ Xq, int64_t ldx, int64_t M, int64_t K,
                   const void* __restrict__ Wv, int64_t ldw, int64_t N,
                   const float* __restrict__ s, const float* __restrict__ beta_dev,
                   const float* __restrict__ bias, float* __restrict__ Y,
                   int32_t* __restrict__ acc_out) {
  __shared__ uint32_t xs[kSimtBM][kSimtKW + 1];
  __shared__ uint32_t wsm[kSimtBN][kSimtKW + 1];
  const int t = threadIdx.x, tx = t & 15, ty = t >> 4;
  const int64_t m0 = int64_t(blockIdx.y) * kSimtBM, n0 = int64_t(blockIdx.x) * kSimtBN;
  const bool xvec = aligned(Xq, 4) && (ldx & 3) == 0;
  const int8_t* W8 = static_cast<const int8_t*>(Wv);
  const uint8_t* Wp = static_cast<const uint8_t*>(Wv);
  const bool wvec = aligned(Wv, 4) && (ldw & 3) == 0;

  int acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0;

  for (int64_t k0 = 0; k0 < K; k0 += kSimtBK) {
#pragma unroll
    for (int r = 0; r < 5; ++r) {
      const int w = t + 256 * r, row = w / kSimtKW, col = w % kSimtKW;
      xs[row][col] = load_i8x4(Xq, ldx, m0 + row, M, k0 + 4 * col, K, xvec);
    }
    if (kPacked) {
      // 64 rows x 16 packed bytes; thread -> (row, 4 bytes) -> 20 trits -> 5 words
      const int row = t >> 2, q = t & 3;
      const int64_t n = n0 + row, j0 = k0 / 5 + 4 * q;
      uint32_t b4 = 0x79797979u;  // four all-zero-trit bytes (121)
      if (n < N) {
        const uint8_t* p = Wp + n * ldw + j0;
        if (wvec) b4 = *reinterpret_cast<const uint32_t*>(p);
        else b4 = uint32_t(p[0]) | uint32_t(p[1]) << 8 | uint32_t(p[2]) << 16 | uint32_t(p[3]) << 24;
      }
      uint32_t tr[20];
#pragma unroll
      for (int bb = 0; bb < 4; ++bb) {
        int t5[5];
        unpack5_byte((b4 >> (8 * bb)) & 0xFFu, t5);
#pragma unroll
        for (int k = 0; k < 5; ++k) tr[5 * bb + k] = uint32_t(uint8_t(int8_t(t5[k])));
      }
#pragma unroll
      for (int v = 0; v < 5; ++v)
        wsm[row][5 * q + v] = tr[4 * v] | tr[4 * v + 1] << 8 | tr[4 * v + 2] << 16 | tr[4 * v + 3] << 24;
    } else {
#pragma unroll
      for (int r = 0; r < 5; ++r) {
        const int w = t + 256 * r, row = w / kSimtKW, col = w % kSimtKW;
        wsm[row][col] = load_i8x4(W8, ldw, n0 + row, N, k0 + 4 * col, K, wvec);
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int kw = 0; kw < kSimtKW; ++kw) {
      int a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = int(xs[ty * 4 + i][kw]);
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = int(wsm[tx * 4 + j][kw]);
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __dp4a(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

  const float beta = kDequant ? *beta_dev : 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t m = m0 + ty * 4 + i;
    if (m >= M) continue;
    const float sb = kDequant ? __fmul_rn(s[m], beta) : 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 4 + j;
      if (n >= N) continue;
      if (kDequant) {
        float y = __fmul_rn(float(acc[i][j]), sb);
        if (bias) y = __fadd_rn(y, bias[n]);
        Y[m * N + n] = y;
      } else {
        acc_out[m * N + n] = acc[i][j];
      }
    }
  }
}

}  // namespace bl
