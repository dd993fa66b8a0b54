// Tensor-core BitLinear for M >= 128 tokens: tcgen05.mma kind::i8 into TMEM.
//
// acc = x_q W_q^T is an exact int8 x int8 -> int32 contraction (the trits are the
// int8 values -1, 0, +1), then y = float32(acc) (s_m beta) [+ b_n]: the deployed-
// path equation of "ultragraph -- when the graph is the 1-bit LLM, part 2",
// section "autograd on a byte-graph".  With many token rows the layer is a dense
// GEMM, so it runs on the 5th-generation tensor cores:
//
//   * a 128 x 256 output tile per CTA, K staged 128 bytes at a time;
//   * TMA (tensor maps, 128-byte swizzle) brings A = X_q [128 x 128] and
//     B = W_q [256 x 128] tiles into a 4-stage shared-memory ring;
//   * one thread issues tcgen05.mma (M=128, N=256, K=32 per instruction, four
//     per stage) accumulating into 256 TMEM columns, and tcgen05.commit frees
//     each stage when its MMAs retire;
//   * the epilogue: each of the 4 warps reads its 32 TMEM lanes (tile rows) with
//     tcgen05.ld, multiplies by s_m * beta (rounded first), adds the bias, and
//     stores float32 Y.  Integer accumulation is exact, so Y matches every other
//     path bit for bit.
//
// Every wait is bounded; on a timeout the kernel records kDevTimeout, waits
// (bounded) for its own in-flight work and frees its TMEM before returning.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kTcBM = 128, kTcBN = 256, kTcBK = 128;
constexpr int kTcStages = 4;
constexpr int kTcStageA = kTcBM * kTcBK;             // 16 KB
constexpr int kTcStageB = kTcBN * kTcBK;             // 32 KB
constexpr int kTcSmem = kTcStages * (kTcStageA + kTcStageB) + 1024;  // + alignment slack
constexpr int kTcThreads = 128;
constexpr uint32_t kTcTmemCols = 256;

struct alignas(64) TcMaps {
  CUtensorMap a;   // X_q [M, K] int8, row stride ldx
  CUtensorMap b;   // W_q [N, K] int8, row stride ldw
};

struct TcArgs {
  int64_t M, N, K;
  const float* s;      // row scales (dequant) or nullptr
  const float* beta;
  const float* bias;
  float* Y;            // [M, N] float32, or nullptr
  int32_t* acc;        // [M, N] int32 when Y is nullptr
};

template <bool kDequant>
__global__ void __launch_bounds__(kTcThreads, 1)
gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t full[kTcStages], empty[kTcStages], tmem_full;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;   // 1024-byte aligned tiles
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  const int64_t m0 = int64_t(blockIdx.y) * kTcBM, n0 = int64_t(blockIdx.x) * kTcBN;
  const int nkb = int(ceil_div(a.K, kTcBK));

  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tmem_full, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.a);
    prefetch_tmap(&maps.b);
  }
  if (warp == 0) {
    tmem_alloc(&s_tmem, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0 && lane == 0) {
    // TMA producer
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % kTcStages;
      if (kb >= kTcStages && !mbar_wait(&empty[s], uint32_t(kb / kTcStages - 1) & 1u)) {
        s_err = 1;
        break;
      }
      unsigned char* sa = smem + s * (kTcStageA + kTcStageB);
      mbar_arrive_expect_tx(&full[s], uint32_t(kTcStageA + kTcStageB));
      tma_load_2d(sa, &maps.a, kb * kTcBK, int(m0), &full[s]);
      tma_load_2d(sa + kTcStageA, &maps.b, kb * kTcBK, int(n0), &full[s]);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    constexpr uint32_t idesc = umma_idesc_i8(kTcBM, kTcBN);
    int kb = 0;
    for (; kb < nkb; ++kb) {
      const int s = kb % kTcStages;
      if (!mbar_wait(&full[s], uint32_t(kb / kTcStages) & 1u)) {
        s_err = 1;
        break;
      }
      tc_fence_after();
      const uint32_t sa = base + uint32_t(s * (kTcStageA + kTcStageB));
      const uint32_t sb = sa + uint32_t(kTcStageA);
#pragma unroll
      for (int k = 0; k < kTcBK / 32; ++k)
        umma_i8(tmem, umma_desc_k_sw128(sa + 32u * k), umma_desc_k_sw128(sb + 32u * k), idesc,
                (kb > 0 || k > 0) ? 1u : 0u);
      umma_commit(&empty[s]);      // the stage is free once these MMAs retire
    }
    umma_commit(&tmem_full);       // all issued MMAs (and the accumulator) are done
  }

  // Epilogue: every warp waits for the accumulator, then drains its 32 lanes.
  const bool done = mbar_wait(&tmem_full, 0u);
  if (!__syncthreads_and(done) || s_err) {
    if (tid == 0) raise_status(kDevTimeout);
  } else {
    tc_fence_after();
    const int row = (warp & 3) * 32 + lane;
    const int64_t m = m0 + row;
    const uint32_t taddr = tmem + (uint32_t((warp & 3) * 32) << 16);
    float sbm = 0.f;
    if (kDequant && m < a.M) sbm = __fmul_rn(a.s[m], *a.beta);
    const bool vec = kDequant ? (aligned(a.Y, 16) && (a.N & 3) == 0) : (aligned(a.acc, 16) && (a.N & 3) == 0);
#pragma unroll 1
    for (int c = 0; c < kTcBN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(taddr + uint32_t(c * 32), r);
      tmem_ld_wait();
      const int64_t nb = n0 + c * 32;
      if (m >= a.M || nb >= a.N) continue;
      if (kDequant) {
        float* yr = a.Y + m * a.N + nb;
        float y[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          y[j] = __fmul_rn(float(int(r[j])), sbm);
          if (a.bias && nb + j < a.N) y[j] = __fadd_rn(y[j], a.bias[nb + j]);
        }
        if (vec && nb + 32 <= a.N) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(yr + j) = make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]);
        } else {
          for (int j = 0; j < 32 && nb + j < a.N; ++j) yr[j] = y[j];
        }
      } else {
        int32_t* ar = a.acc + m * a.N + nb;
        if (vec && nb + 32 <= a.N) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<int4*>(ar + j) = make_int4(int(r[j]), int(r[j + 1]), int(r[j + 2]), int(r[j + 3]));
        } else {
          for (int j = 0; j < 32 && nb + j < a.N; ++j) ar[j] = int(r[j]);
        }
      }
    }
  }
  // Teardown: no MMA may still write TMEM when it is freed.
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTcTmemCols);
  }
}

// W_q from the packed format into int8 rows [N, ldq] for the TMA loads: one
// thread per 4 packed bytes (20 trits); trits at or past K are not written.
__global__ void __launch_bounds__(256)
unpack5_rows_kernel(const uint8_t* __restrict__ Wp, int64_t N, int64_t K, int64_t ldp,
                    int8_t* __restrict__ Wq, int64_t ldq) {
  const int64_t words = ceil_div(ceil_div(K, 5), 4);
  const int64_t total = N * words;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t row = i / words, g = i - row * words;
    const uint32_t w = *reinterpret_cast<const uint32_t*>(Wp + row * ldp + 4 * g);
    uint32_t t[20];
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      int t5[5];
      unpack5_byte((w >> (8 * b)) & 0xFFu, t5);
#pragma unroll
      for (int k = 0; k < 5; ++k) t[5 * b + k] = uint32_t(uint8_t(int8_t(t5[k])));
    }
    int8_t* out = Wq + row * ldq + 20 * g;
    const int64_t k0 = 20 * g;
    if (k0 + 20 <= K) {
#pragma unroll
      for (int v = 0; v < 5; ++v)
        reinterpret_cast<uint32_t*>(out)[v] =
            t[4 * v] | t[4 * v + 1] << 8 | t[4 * v + 2] << 16 | t[4 * v + 3] << 24;
    } else {
      for (int k = 0; k < 20 && k0 + k < K; ++k) out[k] = int8_t(t[k]);
    }
  }
}

}  // namespace bl
