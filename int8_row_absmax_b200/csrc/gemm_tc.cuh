// Tensor-core BitLinear for M >= 128 tokens: tcgen05.mma kind::i8 into TMEM.
//
// acc = x_q W_q^T is an exact int8 x int8 -> int32 contraction (the trits are the
// int8 values -1, 0, +1), then y = float32(acc) (s_m beta) [+ b_n]: the deployed-
// path equation of "ultragraph -- when the graph is the 1-bit LLM, part 2",
// section "autograd on a byte-graph".  With many token rows the layer is a dense
// GEMM, so it runs on the 5th-generation tensor cores.
//
// Persistent kernel, one CTA per SM walking 128 x kBN output tiles (kBN = 256,
// or 64 when 256-wide tiles would leave SMs idle):
//   * warp 0 (one thread): TMA loads of A = X_q [128 x 128 B] and B = W_q
//     [kBN x 128 B] tiles (128-byte swizzle) into a 4- (8-) stage shared-memory ring;
//   * warp 1 (one thread): tcgen05.mma, M=128 N=kBN K=32, four per stage, into
//     one of two kBN-column TMEM accumulators; tcgen05.commit releases each
//     stage, and the accumulator once a tile's K loop is done;
//   * warps 2..5: the epilogue, each warp draining its 32 TMEM lanes (tile rows)
//     with tcgen05.ld, y = float32(acc) * (s_m * beta) [+ b_n], float32 stores;
//     it then hands the accumulator back, so the next tile's MMAs overlap this
//     tile's stores.
// Integer accumulation is exact, so Y matches every other path bit for bit.
// Every wait is bounded; on a timeout the kernel records kDevTimeout, lets
// in-flight MMAs retire (bounded) and frees its TMEM before returning.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kTcBM = 128, kTcBN = 256, kTcBK = 128;
constexpr int kTcStageA = kTcBM * kTcBK;             // 16 KB
constexpr int kTcThreads = 192;                       // producer, MMA, 4 epilogue warps
// Tile width kBN = 256 (4 stages of 16 + 32 KB), or 64 when the 256-wide tiles
// would leave SMs idle (small M: N / 256 tiles only; 8 stages of 16 + 8 KB).
template <int kBN>
struct TcCfg {
  static constexpr int kStages = kBN == 256 ? 4 : 8;
  static constexpr int kStageB = kBN * kTcBK;
  static constexpr int kSmem = kStages * (kTcStageA + kStageB) + 1024;   // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * kBN;                         // two accumulators
};

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
  int tiles_m, tiles_n;
};

template <bool kDequant, int kBN = kTcBN>
__global__ void __launch_bounds__(kTcThreads, 1)
gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
  constexpr int kTcStages = TcCfg<kBN>::kStages;
  constexpr int kTcStageB = TcCfg<kBN>::kStageB;
  constexpr uint32_t kTcTmemCols = TcCfg<kBN>::kTmemCols;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t full[kTcStages], empty[kTcStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* err = &s_err;                                     // polled across roles
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;   // 1024-byte aligned tiles
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  const int nkb = int(ceil_div(a.K, kTcBK));
  const int ntiles = a.tiles_m * a.tiles_n;

  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);     // one arrive per epilogue warp
    }
    mbar_init(&drain, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.a);
    prefetch_tmap(&maps.b);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, kTcTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      // TMA producer: the stage ring runs continuously across tiles
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && !*err; t += gridDim.x) {
        const int tm = t / a.tiles_n, tn = t - tm * a.tiles_n;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kTcStages;
          if (it >= kTcStages && !mbar_wait(&empty[s], uint32_t(it / kTcStages - 1) & 1u)) {
            *err = 1;
            break;
          }
          unsigned char* sa = smem + s * (kTcStageA + kTcStageB);
          mbar_arrive_expect_tx(&full[s], uint32_t(kTcStageA + kTcStageB));
          tma_load_2d(sa, &maps.a, kb * kTcBK, tm * kTcBM, &full[s]);
          tma_load_2d(sa + kTcStageA, &maps.b, kb * kTcBK, tn * kBN, &full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // MMA issuer
      constexpr uint32_t idesc = umma_idesc_i8(kTcBM, kBN);
      int it = 0, u = 0;
      for (int t = blockIdx.x; t < ntiles && !*err; t += gridDim.x, ++u) {
        const int b = u & 1;
        if (u >= 2 && !mbar_wait(&acc_empty[b], uint32_t(u / 2 - 1) & 1u)) {
          *err = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(b * kBN);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % kTcStages;
          if (!mbar_wait(&full[s], uint32_t(it / kTcStages) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + uint32_t(s * (kTcStageA + kTcStageB));
          const uint32_t sb = sa + uint32_t(kTcStageA);
#pragma unroll
          for (int k = 0; k < kTcBK / 32; ++k)
            umma_i8(d, umma_desc_k_sw128(sa + 32u * k), umma_desc_k_sw128(sb + 32u * k), idesc,
                    (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[s]);    // the stage is free once these MMAs retire
        }
        umma_commit(&acc_full[b]);   // the accumulator is complete (or abandoned)
        if (!ok) {
          *err = 1;
          break;
        }
      }
      umma_commit(&drain);           // every MMA issued by this thread has retired
    }
  } else {
    // epilogue warps 2..5: warp w owns TMEM lanes 32*(w%4) .. +31
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool vec = kDequant ? (aligned(a.Y, 16) && (a.N & 3) == 0) : (aligned(a.acc, 16) && (a.N & 3) == 0);
    const float beta = kDequant ? *a.beta : 0.f;
    int u = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++u) {
      const int b = u & 1;
      if (!mbar_wait(&acc_full[b], uint32_t(u / 2) & 1u)) {
        *err = 1;
        break;
      }
      if (*err) break;
      tc_fence_after();
      const int tm = t / a.tiles_n, tn = t - tm * a.tiles_n;
      const int64_t m = int64_t(tm) * kTcBM + row;
      const int64_t n0 = int64_t(tn) * kBN;
      const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + uint32_t(b * kBN);
      float sbm = 0.f;
      if (kDequant && m < a.M) sbm = __fmul_rn(a.s[m], beta);
#pragma unroll 1
      for (int c = 0; c < kBN / 32; ++c) {
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
              *reinterpret_cast<int4*>(ar + j) =
                  make_int4(int(r[j]), int(r[j + 1]), int(r[j + 2]), int(r[j + 3]));
          } else {
            for (int j = 0; j < 32 && nb + j < a.N; ++j) ar[j] = int(r[j]);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&acc_empty[b]);   // this warp is done with accumulator b
    }
  }

  // Teardown: the MMA thread's last commit must have landed before TMEM is freed.
  __syncthreads();
  if (warp == 1) {
    const bool drained = mbar_wait(&drain, 0u);
    if ((!drained || *err) && lane == 0) raise_status(kDevTimeout);
    __syncwarp();
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
  const bool small = total < (int64_t(1) << 32);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    int64_t row, g;
    split_index(i, words, small, row, g);
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
