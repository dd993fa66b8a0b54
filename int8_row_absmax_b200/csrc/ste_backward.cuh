// Straight-through backward of the BitLinear layer on the tensor cores.
//
// "ultragraph -- when the graph is the 1-bit LLM, part 2", section "autograd on
// a byte-graph, and the straight-through lie": the quantizers and the per-row
// scale count as the identity on the way back, so the gradients reach the
// float32 masters through two dense products and a column sum:
//     dX = dY W  [M, K],     dW = dY^T X  [N, K],     db = sum over rows of dY  [N].
//
// Both products run as D[r, c] = sum_j A[r, j] B[c, j] on tcgen05 (kind::tf32,
// float32 accumulators in TMEM), with A and B K-major (the contraction index j
// contiguous).  A tf32 operand keeps 11 significant bits, so each float32
// operand is split as a = a_hi + a_lo with a_hi = tf32(a) and a_lo = tf32(a -
// a_hi) (a - a_hi is exact in float32), and each product is taken as
// a_hi b_hi + a_hi b_lo + a_lo b_hi: three MMAs into the same accumulator.
// The dropped a_lo b_lo and the rounding of the lo parts leave at most about
// 3 * 2^-22 |a b| per product, on the order of float32's own rounding (the
// published "3xTF32" split).
//
//   split_tf32_kernel   float32 [R, C] -> hi, lo [R, ld] (or transposed [C, ld]),
//                       zero padding up to ld (a multiple of 4: 16-byte TMA rows);
//                       the transposing form goes through a 32 x 33 shared tile;
//   gemm_tf32x3_kernel  persistent, one CTA per SM, 128 x 256 output tiles; warp 0
//                       issues the TMA loads (four tiles per K block: A_hi, A_lo,
//                       B_hi, B_lo, 128-byte swizzle), warp 1 the MMAs (4 K steps
//                       of 8 x 3 products per block) into one of two 256-column
//                       accumulators, warps 2..5 drain TMEM into float32 D;
//   colsum_kernel       db[n] = float32(sum_m dY[m, n]) accumulated in float64.
// Every wait is bounded; a timeout records kDevTimeout and the kernel lets the
// MMAs in flight land and frees its TMEM before returning.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kBwBM = 128, kBwBN = 256, kBwBK = 32;          // K block: 32 float32 = 128 bytes
constexpr int kBwTileA = kBwBM * kBwBK * 4;                   // 16 KB
constexpr int kBwTileB = kBwBN * kBwBK * 4;                   // 32 KB
constexpr int kBwStage = 2 * kBwTileA + 2 * kBwTileB;         // A_hi, A_lo, B_hi, B_lo: 96 KB
constexpr int kBwStages = 2;
constexpr int kBwSmem = kBwStages * kBwStage + 1024;
constexpr int kBwThreads = 192;
constexpr uint32_t kBwTmemCols = 2 * kBwBN;

// tf32 rounding of a float32 (round to nearest, ties away; low 13 bits zero).
__device__ __forceinline__ float tf32_round(float a) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(a));
  return __uint_as_float(r);
}

// hi/lo split of src [R, C] (row stride lds floats) into [R, ld] (kTrans = false)
// or [C, ld] (kTrans = true), columns past the source extent zero.
template <bool kTrans>
__global__ void __launch_bounds__(256)
split_tf32_kernel(const float* __restrict__ src, int64_t R, int64_t C, int64_t lds, float* __restrict__ hi,
                  float* __restrict__ lo, int64_t ld) {
  if (!kTrans) {
    const int64_t total = R * ld;
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += int64_t(gridDim.x) * blockDim.x) {
      const int64_t r = i / ld, c = i - r * ld;
      const float a = c < C ? src[r * lds + c] : 0.f;
      const float h = tf32_round(a);
      hi[i] = h;
      lo[i] = tf32_round(__fsub_rn(a, h));
    }
    return;
  }
  // transposed: output row c holds column c of src; 32 x 32 tiles.  Output
  // columns run to ld (source rows R..ld-1 are the zero padding).
  __shared__ float tile[32][33];
  const int64_t nbi = ceil_div(ld, 32), nbj = ceil_div(C, 32);
  for (int64_t t = blockIdx.x; t < nbi * nbj; t += gridDim.x) {
    const int64_t bi = t / nbj, bj = t - bi * nbj;   // source row block bi (output cols), column block bj
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;   // 8 rows of 32 per pass
    for (int y = ty; y < 32; y += 8) {
      const int64_t r = bi * 32 + y, c = bj * 32 + tx;           // read src[r, c]
      tile[y][tx] = (r < R && c < C) ? src[r * lds + c] : 0.f;
    }
    __syncthreads();
    for (int y = ty; y < 32; y += 8) {
      const int64_t oc = bj * 32 + y, orr = bi * 32 + tx;        // out[oc, orr] = src[orr, oc]
      if (oc < C && orr < ld) {
        const float a = tile[tx][y];
        const float h = tf32_round(a);
        hi[oc * ld + orr] = h;
        lo[oc * ld + orr] = tf32_round(__fsub_rn(a, h));
      }
    }
    __syncthreads();
  }
}

// db[n] = float32(sum_m dY[m, n]), each column summed in float64 by one thread
// (consecutive threads take consecutive columns: coalesced rows).
__global__ void __launch_bounds__(256)
colsum_kernel(const float* __restrict__ dY, int64_t M, int64_t N, float* __restrict__ db) {
  for (int64_t n = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; n < N; n += int64_t(gridDim.x) * blockDim.x) {
    double s = 0.0;
    for (int64_t m = 0; m < M; ++m) s += double(dY[m * N + n]);
    db[n] = float(s);
  }
}

struct alignas(64) BwMaps {
  CUtensorMap a_hi, a_lo, b_hi, b_lo;   // float32 [rows, Kc], K-major, 128-byte swizzle
};

struct BwArgs {
  int64_t Mr, Nc, Kc;    // D is [Mr, Nc]; contraction over Kc
  float* D;              // row-major, row stride Nc
  int tiles_m, tiles_n;
};

// Instruction descriptor, kind::tf32: float32 accumulator, A and B tf32 and K-major.
__host__ __device__ constexpr uint32_t umma_idesc_tf32(int m, int n) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (uint32_t(n >> 3) << 17) | (uint32_t(m >> 4) << 24);
}

__device__ __forceinline__ void umma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kBwThreads, 1)
gemm_tf32x3_kernel(const __grid_constant__ BwMaps maps, const BwArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t full[kBwStages], empty[kBwStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* err = &s_err;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  const int nkb = int(ceil_div(a.Kc, kBwBK));
  const int nwork = a.tiles_m * a.tiles_n;

  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < kBwStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(&drain, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.a_hi);
    prefetch_tmap(&maps.a_lo);
    prefetch_tmap(&maps.b_hi);
    prefetch_tmap(&maps.b_lo);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kBwTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      int it = 0;
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x) {
        const int tm = w / a.tiles_n, tn = w - tm * a.tiles_n;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kBwStages;
          if (it >= kBwStages && !mbar_wait(&empty[s], uint32_t(it / kBwStages - 1) & 1u)) {
            *err = 1;
            break;
          }
          unsigned char* st = smem + s * kBwStage;
          mbar_arrive_expect_tx(&full[s], uint32_t(kBwStage));
          tma_load_2d(st, &maps.a_hi, kb * kBwBK, tm * kBwBM, &full[s]);
          tma_load_2d(st + kBwTileA, &maps.a_lo, kb * kBwBK, tm * kBwBM, &full[s]);
          tma_load_2d(st + 2 * kBwTileA, &maps.b_hi, kb * kBwBK, tn * kBwBN, &full[s]);
          tma_load_2d(st + 2 * kBwTileA + kBwTileB, &maps.b_lo, kb * kBwBK, tn * kBwBN, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc_tf32(kBwBM, kBwBN);
      int it = 0, u = 0;
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x, ++u) {
        const int b = u & 1;
        if (u >= 2 && !mbar_wait(&acc_empty[b], uint32_t(u / 2 - 1) & 1u)) {
          *err = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(b * kBwBN);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kBwStages;
          if (!mbar_wait(&full[s], uint32_t(it / kBwStages) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ah = base + uint32_t(s * kBwStage);
          const uint32_t al = ah + uint32_t(kBwTileA);
          const uint32_t bh = ah + uint32_t(2 * kBwTileA);
          const uint32_t blo = bh + uint32_t(kBwTileB);
#pragma unroll
          for (int k = 0; k < kBwBK / 8; ++k) {            // 8 tf32 = 32 bytes per MMA
            const uint32_t off = 32u * uint32_t(k);
            umma_tf32(d, umma_desc_k_sw128(ah + off), umma_desc_k_sw128(bh + off), idesc,
                      (kb > 0 || k > 0) ? 1u : 0u);
            umma_tf32(d, umma_desc_k_sw128(ah + off), umma_desc_k_sw128(blo + off), idesc, 1u);
            umma_tf32(d, umma_desc_k_sw128(al + off), umma_desc_k_sw128(bh + off), idesc, 1u);
          }
          umma_commit(&empty[s]);
        }
        umma_commit(&acc_full[b]);
        if (!ok) {
          *err = 1;
          break;
        }
      }
      umma_commit(&drain);
    }
  } else {
    // epilogue warps 2..5: warp w owns TMEM lanes 32*(w%4) .. +31 (tile rows)
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool vec = aligned(a.D, 16) && (a.Nc & 3) == 0;
    int u = 0;
    for (int w = blockIdx.x; w < nwork; w += gridDim.x, ++u) {
      const int b = u & 1;
      if (!mbar_wait(&acc_full[b], uint32_t(u / 2) & 1u)) {
        *err = 1;
        break;
      }
      if (*err) break;
      tc_fence_after();
      const int tm = w / a.tiles_n, tn = w - tm * a.tiles_n;
      const int64_t m = int64_t(tm) * kBwBM + row;
      const int64_t n0 = int64_t(tn) * kBwBN;
      const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + uint32_t(b * kBwBN);
#pragma unroll 1
      for (int cc = 0; cc < kBwBN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(taddr + uint32_t(cc * 32), r);
        tmem_ld_wait();
        const int64_t nb = n0 + cc * 32;
        if (m >= a.Mr || nb >= a.Nc) continue;
        float* dr = a.D + m * a.Nc + nb;
        if (vec && nb + 32 <= a.Nc) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(dr + j) = make_float4(__uint_as_float(r[j]), __uint_as_float(r[j + 1]),
                                                             __uint_as_float(r[j + 2]), __uint_as_float(r[j + 3]));
        } else {
          for (int j = 0; j < 32 && nb + j < a.Nc; ++j) dr[j] = __uint_as_float(r[j]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);
    }
  }

  __syncthreads();
  if (warp == 1) {
    const bool drained = mbar_wait(&drain, 0u);
    if ((!drained || *err) && lane == 0) raise_status(kDevTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kBwTmemCols);
  }
}

}  // namespace bl
