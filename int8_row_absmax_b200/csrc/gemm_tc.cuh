// Tensor-core BitLinear for M >= 128 tokens: tcgen05.mma kind::i8 into TMEM.
//
// acc = x_q W_q^T is an exact int8 x int8 -> int32 contraction (the trits are the
// int8 values -1, 0, +1), then y = float32(acc) (s_m beta) [+ b_n]: the deployed-
// path equation of "ultragraph -- when the graph is the 1-bit LLM, part 2",
// section "autograd on a byte-graph".  With many token rows the layer is a dense
// GEMM, so it runs on the 5th-generation tensor cores.
//
// Persistent kernel, one CTA per SM walking 128 x kBN output tiles (kBN = 256,
// or 64 when 256-wide tiles would leave SMs idle).  With packed weights
// (kPacked) B never exists as int8 in HBM: TMA brings packed super-tiles (128
// bytes = 640 trits per row, 128-byte swizzle) into a ring of their own, and
// eight decoder warps expand each into five int8 B stages.  Decode: trits
// t0..t3 of a byte come from a shared-memory table with one copy per lane (no
// bank conflicts); t4 = floor(b/81) - 1 is computed for four bytes at once
// (b * 203 in 16-bit lanes holds it in bits 14..15, exact for b <= 242);
// byte_perm cuts the 16-trit window of each 16-byte chunk, which is stored at
// the int8 stage's 128-byte-swizzle position; then fence.proxy.async and an
// arrive on the stage.  Bytes above 242 are not codes: they decode to
// unspecified trits.
// Roles:
//   * warp 0 (one thread): TMA loads of A = X_q [128 x 128 B] and B = W_q
//     [kBN x 128 B] tiles (128-byte swizzle) into a 4- (8-) stage shared-memory
//     ring (packed: A only; warp 14 loads the packed super-tiles, warps 6..13
//     decode them into the B halves of the stages);
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
// With packed weights (kPacked) the B stages are filled by decoder warps from
// packed super-tiles (640 trits = 128 bytes per row): fewer int8 stages, a ring
// of super-tiles deep enough to keep HBM busy when the weights stream once
// (10 x 8 KB for 64-wide tiles; 2 x 32 KB for 256-wide ones), and the 32 KB
// decode table.
constexpr int kTpDecWarps = 8;
constexpr int kTpSuper = 5;                           // int8 K blocks per packed super-tile
template <int kBN, bool kPacked = false>
struct TcCfg {
  static constexpr int kStages = kPacked ? (kBN == 256 ? 2 : 4) : (kBN == 256 ? 4 : 8);
  static constexpr int kStageB = kBN * kTcBK;
  static constexpr int kPkStages = kPacked ? (kBN == 256 ? 2 : 10) : 1;
  static constexpr int kPkBytes = kPacked ? kBN * 128 : 0;
  static constexpr int kLutBytes = kPacked ? 256 * 128 : 0;   // word 32 b + lane: t0..t3 of byte b
  static constexpr int kSmem =
      kStages * (kTcStageA + kStageB) + kPkStages * kPkBytes + kLutBytes + 1024;  // + alignment slack
  static constexpr uint32_t kTmemCols = 2 * kBN;                         // two accumulators
  // packed: + the decoder warps and one warp that issues the packed loads
  static constexpr int kThreads = kTcThreads + (kPacked ? 32 * (kTpDecWarps + 1) : 0);
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

template <bool kDequant, int kBN = kTcBN, bool kPacked = false>
__global__ void __launch_bounds__(TcCfg<kBN, kPacked>::kThreads, 1)
gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
  constexpr int kTcStages = TcCfg<kBN, kPacked>::kStages;
  constexpr int kTcStageB = TcCfg<kBN, kPacked>::kStageB;
  constexpr int kPkBytes = TcCfg<kBN, kPacked>::kPkBytes;
  constexpr int kPkStages = TcCfg<kBN, kPacked>::kPkStages;
  constexpr uint32_t kTcTmemCols = TcCfg<kBN, kPacked>::kTmemCols;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t full[kTcStages], empty[kTcStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint64_t pk_full[kPkStages], pk_empty[kPkStages];
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* err = &s_err;                                     // polled across roles
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;   // 1024-byte aligned tiles
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  const int nkb = int(ceil_div(a.K, kTcBK));
  const int ntiles = a.tiles_m * a.tiles_n;
  unsigned char* pk = smem + kTcStages * (kTcStageA + kTcStageB);   // packed ring (kPacked)
  uint32_t* lut = reinterpret_cast<uint32_t*>(pk + kPkStages * kPkBytes);
  if (kPacked) {
    // word 32 b + l: digits d0..d3 of byte b (b = sum d_k 3^k), each as the
    // int8 trit d_k - 1; bytes past 242 read as 121 (all zero) here
    for (int w = tid; w < 256 * 32; w += blockDim.x) {
      uint32_t x = uint32_t(w >> 5), v = 0;
      if (x > 242u) x = 121u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v |= ((x % 3u + 255u) & 0xFFu) << (8 * k);
        x /= 3u;
      }
      lut[w] = v;
    }
  }

  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1 + (kPacked ? kTpDecWarps : 0));   // (+ one arrive per decoder warp)
      mbar_init(&empty[s], 1);
    }
    for (int p = 0; p < (kPacked ? kPkStages : 0); ++p) {
      mbar_init(&pk_full[p], 1);
      mbar_init(&pk_empty[p], kTpDecWarps);
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
          if (kPacked) {
            mbar_arrive_expect_tx(&full[s], uint32_t(kTcStageA));
            tma_load_2d(sa, &maps.a, kb * kTcBK, tm * kTcBM, &full[s]);
          } else {
            mbar_arrive_expect_tx(&full[s], uint32_t(kTcStageA + kTcStageB));
            tma_load_2d(sa, &maps.a, kb * kTcBK, tm * kTcBM, &full[s]);
            tma_load_2d(sa + kTcStageA, &maps.b, kb * kTcBK, tn * kBN, &full[s]);
          }
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
  } else if (kPacked && warp == 6 + kTpDecWarps) {
    if (lane == 0) {
      // packed producer: super-tiles (rows tn*kBN.., bytes 128 j.., 640 trits)
      // run ahead of the decoders by up to kPkStages, across tiles, independent
      // of the int8 stage ring
      int pj = 0;
      for (int t = blockIdx.x; t < ntiles && !*err; t += gridDim.x) {
        const int tn = t % a.tiles_n;
        for (int kb0 = 0; kb0 < nkb; kb0 += kTpSuper, ++pj) {
          const int p = pj % kPkStages;
          if (pj >= kPkStages && !mbar_wait(&pk_empty[p], uint32_t(pj / kPkStages - 1) & 1u)) {
            *err = 1;
            break;
          }
          mbar_arrive_expect_tx(&pk_full[p], uint32_t(kPkBytes));
          tma_load_2d(pk + p * kPkBytes, &maps.b, (kb0 / kTpSuper) * 128, tn * kBN, &pk_full[p]);
        }
      }
      // copies still in flight (after an error) land before the CTA exits
      for (int q = pj > kPkStages ? pj - kPkStages : 0; q < pj; ++q)
        (void)mbar_wait(&pk_full[q % kPkStages], uint32_t(q / kPkStages) & 1u);
    }
  } else if (kPacked && warp >= 6) {
    // decoder warps: thread dt owns 16-byte chunk c = dt % 8 of rows dt / 8 + 32 i
    // of each B stage (K-major, 128-byte swizzle: chunk c of row r at
    // r * 128 + (c ^ (r % 8)) * 16; r % 8 = sw for all of this thread's rows)
    const int dt = tid - 6 * 32;
    const uint32_t c = uint32_t(dt & 7), sw = uint32_t(dt >> 3) & 7u;
    const uint32_t* lut_l = lut + lane;
    int it = 0, pj = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok && !*err; t += gridDim.x) {
      for (int kb0 = 0; kb0 < nkb; kb0 += kTpSuper, ++pj) {
        const int p = pj % kPkStages;
        if (!mbar_wait(&pk_full[p], uint32_t(pj / kPkStages) & 1u)) {
          ok = false;
          break;
        }
        const unsigned char* src = pk + p * kPkBytes + (dt >> 3) * 128;
#pragma unroll
        for (int sub = 0; sub < kTpSuper; ++sub) {
          if (kb0 + sub >= nkb) break;
          const int s = it % kTcStages;
          if (it >= kTcStages && !mbar_wait(&empty[s], uint32_t(it / kTcStages - 1) & 1u)) {
            ok = false;
            break;
          }
          // the chunk's 16 trits start at trit t0 of the super-tile row: packed
          // bytes b0..b0+3 hold them after al leading trits
          const uint32_t t0 = 128u * uint32_t(sub) + 16u * c;
          const uint32_t b0 = (t0 * 52429u) >> 18, al = t0 - 5u * b0;   // t0 / 5, t0 % 5
          const uint32_t w0 = b0 >> 2, w1 = w0 < 31u ? w0 + 1u : 31u;
          // the packed tile has the 128-byte swizzle too (row % 8 = sw)
          const uint32_t o0 = (((w0 >> 2) ^ sw) << 4) | ((w0 & 3u) << 2);
          const uint32_t o1 = (((w1 >> 2) ^ sw) << 4) | ((w1 & 3u) << 2);
          const uint32_t sh = 8u * (b0 & 3u), sel = 0x3210u + 0x1111u * al;
          unsigned char* dst = smem + s * (kTcStageA + kTcStageB) + kTcStageA + (dt >> 3) * 128 + ((c ^ sw) << 4);
#pragma unroll
          for (int i = 0; i < kBN / 32; ++i) {
            const unsigned char* row = src + i * 32 * 128;
            const uint32_t four = __funnelshift_r(*reinterpret_cast<const uint32_t*>(row + o0),
                                                  *reinterpret_cast<const uint32_t*>(row + o1), sh);
            const uint32_t L0 = lut_l[(four & 0xFFu) << 5], L1 = lut_l[((four >> 8) & 0xFFu) << 5];
            const uint32_t L2 = lut_l[((four >> 16) & 0xFFu) << 5], L3 = lut_l[(four >> 24) << 5];
            // t4 of the four bytes: the top two bits of each byte's b * 203 (16-bit lanes)
            const uint32_t lo = (four & 0x00FF00FFu) * 203u, hi = ((four >> 8) & 0x00FF00FFu) * 203u;
            const uint32_t T = (((__byte_perm(lo, hi, 0x7351) >> 6) & 0x03030303u) + 0x7F7F7F7Fu) ^ 0x80808080u;
            // the 20 trits of the four bytes in order, then the 16 starting at al
            const uint32_t S0 = L0, S1 = __byte_perm(T, L1, 0x6540);
            const uint32_t S2 = __byte_perm(__byte_perm(L1, T, 0x0053), L2, 0x5410);
            const uint32_t S3 = __byte_perm(__byte_perm(L2, T, 0x0632), L3, 0x4210);
            const uint32_t S4 = __byte_perm(L3, T, 0x7321);
            *reinterpret_cast<uint4*>(dst + i * 32 * 128) =
                make_uint4(__byte_perm(S0, S1, sel), __byte_perm(S1, S2, sel), __byte_perm(S2, S3, sel),
                           __byte_perm(S3, S4, sel));
          }
          fence_proxy_async_smem();      // generic-proxy writes, read by the tensor cores
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
          ++it;
        }
        if (!ok) break;
        if (lane == 0) mbar_arrive(&pk_empty[p]);   // every lane's reads precede the last __syncwarp
      }
    }
    if (!ok) *err = 1;
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
