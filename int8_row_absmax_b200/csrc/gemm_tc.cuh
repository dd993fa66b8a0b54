// Tensor-core BitLinear: tcgen05.mma kind::i8 into TMEM.
//
// acc = x_q W_q^T is an exact int8 x int8 -> int32 contraction (the trits are the
// int8 values -1, 0, +1), then y = float32(acc) (s_m beta) [+ b_n]: the deployed-
// path equation of "ultragraph -- when the graph is the 1-bit LLM, part 2",
// section "autograd on a byte-graph".  With several token rows the layer is a
// dense GEMM, so it runs on the 5th-generation tensor cores.
//
// Persistent kernel, one CTA per SM, walking work items: a 128 x 256 output
// tile over a range of K.  An int8 MMA of 128 rows x 32 K takes about as long
// at N = 64 as at N = 256 (measured), so tiles are always 256 wide.  When there
// are fewer tiles than SMs, K is split into `split` ranges of whole 640-wide
// chunks; each split writes its int32 partial tile to the workspace and
// tc_reduce_kernel adds them up and runs the epilogue's arithmetic.  Integer
// partial sums are exact, so splitting changes no bit of the result.
//
// With packed weights (kPacked) B never exists as int8 in HBM: TMA brings
// packed chunks (128 bytes = 640 trits per row, 128-byte swizzle) into a ring
// of their own, and sixteen decoder warps expand them into the int8 B stages.
// Decode: trits t0..t3 of a byte come from a shared-memory table with one copy
// per lane (no bank conflicts); t4 = floor(b/81) - 1 is computed for four bytes
// at once (b * 203 in 16-bit lanes holds it in bits 14..15, exact for b <= 242);
// byte_perm cuts the 16-trit window of each 16-byte chunk, which is stored at
// the int8 stage's 128-byte-swizzle position; then fence.proxy.async and an
// arrive on the stage.  The decoder warps form two groups that take the K
// blocks in turn, so two blocks are in decode at once and each thread has
// eight independent chunks per block (fewer left the decoders latency-bound).
// Bytes above 242 are not codes: they decode to unspecified trits.
// Roles:
//   * warp 0 (one thread): TMA loads of A = X_q [128 x 128 B] and (int8 weights)
//     B = W_q [256 x 128 B] tiles, 128-byte swizzle, into the stage ring;
//   * warp 1 (one thread): tcgen05.mma, M=128 N=256 K=32, four per stage, into
//     one of two 256-column TMEM accumulators; tcgen05.commit releases each
//     stage, and the accumulator once a work item's K loop is done;
//   * warps 2..5: the epilogue, each warp draining its 32 TMEM lanes (tile rows)
//     with tcgen05.ld, y = float32(acc) * (s_m * beta) [+ b_n], float32 stores;
//     it then hands the accumulator back, so the next item's MMAs overlap this
//     item's stores;
//   * packed: warps 6..21 decode, warp 22 (one thread) loads the packed chunks.
// Every wait is bounded; on a timeout the kernel records kDevTimeout, lets
// in-flight MMAs and packed copies land (bounded) and frees its TMEM.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "trit_table.cuh"

namespace bl {

constexpr int kTcBM = 128, kTcBN = 256, kTcBK = 128;
constexpr int kTcStageA = kTcBM * kTcBK;             // 16 KB
constexpr int kTcStageB = kTcBN * kTcBK;             // 32 KB
constexpr int kTcThreads = 192;                       // producer, MMA, 4 epilogue warps
constexpr int kTcChunk = 5;                           // K blocks per chunk: 640 trits = 128 packed bytes
constexpr int kTcMaxSplit = 8;
constexpr uint32_t kTcTmemCols = 2 * kTcBN;           // two accumulators
constexpr int kTpDecWarps = 16, kTpDecGroups = 2;
constexpr int kTpWpg = kTpDecWarps / kTpDecGroups;    // decoder warps per group
constexpr int kTpPkWarp = kTcThreads / 32 + kTpDecWarps;
constexpr int kTpDecBar = 1;                          // named barrier of the decoder warps
// int8 weights: 4 stages of 16 + 32 KB.  Packed: 2 stages, a ring of two packed
// chunks (32 KB each) and the 32 KB decode table (word 32 b + lane: t0..t3 of b).
template <bool kPacked>
struct TcCfg {
  static constexpr int kStages = kPacked ? 2 : 4;
  static constexpr int kPkStages = kPacked ? 2 : 1;
  static constexpr int kPkBytes = kPacked ? kTcBN * 128 : 0;
  static constexpr int kLutBytes = kPacked ? 256 * 128 : 0;
  static constexpr int kSmem =
      kStages * (kTcStageA + kTcStageB) + kPkStages * kPkBytes + kLutBytes + 1024;  // + alignment slack
  static constexpr int kThreads = kTcThreads + (kPacked ? 32 * (kTpDecWarps + 1) : 0);
};

struct alignas(64) TcMaps {
  CUtensorMap a;   // X_q [M, K] int8, row stride ldx
  CUtensorMap b;   // W_q [N, K] int8, row stride ldw (or packed [N, ldp] bytes)
};

struct TcArgs {
  int64_t M, N, K;
  const float* s;      // row scales (dequant) or nullptr
  const float* beta;
  const float* bias;
  float* Y;            // [M, N] float32, or nullptr
  int32_t* acc;        // [M, N] int32 when Y is nullptr
  int tiles_m, tiles_n;
  int split;           // K ranges per tile (1: no partials)
  int32_t* part;       // [split, M, N] int32 partial sums (split > 1)
};

// Output tile t -> (row tile, column tile), grouped: consecutive tiles walk
// kTcGroupM row tiles down one column of tiles before moving right, so the
// CTAs running at one time share a few A row panels and B column panels and
// the operands they re-read stay in L2.
constexpr int kTcGroupM = 8;
__device__ __forceinline__ void tc_tile_coords(const TcArgs& a, int t, int& tm, int& tn) {
  const int per_group = kTcGroupM * a.tiles_n;
  const int g = t / per_group, r = t - g * per_group;
  const int first = g * kTcGroupM;
  const int gm = min(kTcGroupM, a.tiles_m - first);
  tm = first + r % gm;
  tn = r / gm;
}

// y (or acc) for 32 columns nb.. of row m from the 32 sums r (streaming
// stores: the output is not read again, so it should not push the operands
// out of L2).
template <bool kDequant>
__device__ __forceinline__ void tc_store32(const TcArgs& a, const uint32_t (&r)[32], int64_t m, int64_t nb,
                                           float sbm, bool vec) {
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
        __stcs(reinterpret_cast<float4*>(yr + j), make_float4(y[j], y[j + 1], y[j + 2], y[j + 3]));
    } else {
      for (int j = 0; j < 32 && nb + j < a.N; ++j) yr[j] = y[j];
    }
  } else {
    int32_t* ar = a.acc + m * a.N + nb;
    if (vec && nb + 32 <= a.N) {
#pragma unroll
      for (int j = 0; j < 32; j += 4)
        __stcs(reinterpret_cast<int4*>(ar + j), make_int4(int(r[j]), int(r[j + 1]), int(r[j + 2]), int(r[j + 3])));
    } else {
      for (int j = 0; j < 32 && nb + j < a.N; ++j) ar[j] = int(r[j]);
    }
  }
}

template <bool kDequant, bool kPacked>
__global__ void __launch_bounds__(TcCfg<kPacked>::kThreads, 1)
gemm_tc_kernel(const __grid_constant__ TcMaps maps, const TcArgs a) {
  constexpr int kStages = TcCfg<kPacked>::kStages;
  constexpr int kPkStages = TcCfg<kPacked>::kPkStages;
  constexpr int kPkBytes = TcCfg<kPacked>::kPkBytes;
  constexpr int kBN = kTcBN;
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t full[kStages], empty[kStages], acc_full[2], acc_empty[2], drain;
  __shared__ uint64_t pk_full[kPkStages], pk_empty[kPkStages];
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* err = &s_err;                                     // polled across roles
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;   // 1024-byte aligned tiles
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  unsigned char* pk = smem + kStages * (kTcStageA + kTcStageB);  // packed ring (kPacked)
  uint32_t* lut = reinterpret_cast<uint32_t*>(pk + kPkStages * kPkBytes);
  const int nkb = int(ceil_div(a.K, kTcBK));
  const int nch = int(ceil_div(nkb, kTcChunk));
  const int S = a.split;
  const int nwork = a.tiles_m * a.tiles_n * S;
  // work item w: tile w / S over K blocks [kb0, kb1), the whole chunks
  // [j nch / S, (j + 1) nch / S) of split j = w % S (S <= nch: none is empty)
  auto work = [&](int w, int& t, int& j, int& kb0, int& kb1) {
    t = w / S;
    j = w - t * S;
    kb0 = (j * nch / S) * kTcChunk;
    kb1 = min(((j + 1) * nch / S) * kTcChunk, nkb);
  };

  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1 + (kPacked ? kTpWpg : 0));   // (+ one arrive per warp of the decoding group)
      mbar_init(&empty[s], 1);
    }
    for (int p = 0; p < (kPacked ? kPkStages : 0); ++p) {
      mbar_init(&pk_full[p], 1);
      mbar_init(&pk_empty[p], kTcChunk * kTpWpg);        // per K block, per warp of its group
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
      // TMA producer: the stage ring runs continuously across work items
      int it = 0;
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x) {
        int t, j, kb0, kb1;
        work(w, t, j, kb0, kb1);
        int tm, tn;
        tc_tile_coords(a, t, tm, tn);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % kStages;
          if (it >= kStages && !mbar_wait(&empty[s], uint32_t(it / kStages - 1) & 1u)) {
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
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x, ++u) {
        int t, j, kb0, kb1;
        work(w, t, j, kb0, kb1);
        const int b = u & 1;
        if (u >= 2 && !mbar_wait(&acc_empty[b], uint32_t(u / 2 - 1) & 1u)) {
          *err = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(b * kBN);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % kStages;
          if (!mbar_wait(&full[s], uint32_t(it / kStages) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = base + uint32_t(s * (kTcStageA + kTcStageB));
          const uint32_t sb = sa + uint32_t(kTcStageA);
#pragma unroll
          for (int k = 0; k < kTcBK / 32; ++k)
            umma_i8(d, umma_desc_k_sw128(sa + 32u * k), umma_desc_k_sw128(sb + 32u * k), idesc,
                    (kb > kb0 || k > 0) ? 1u : 0u);
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
  } else if (kPacked && warp == kTpPkWarp) {
    if (lane == 0) {
      // packed producer: chunks (rows tn*256.., bytes 128 c.., 640 trits) run
      // ahead of the decoders by up to kPkStages, independent of the stage ring
      int pj = 0;
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x) {
        int t, j, kb0, kb1;
        work(w, t, j, kb0, kb1);
        int tm, tn;
        tc_tile_coords(a, t, tm, tn);
        for (int c = kb0 / kTcChunk; c * kTcChunk < kb1; ++c, ++pj) {
          const int p = pj % kPkStages;
          if (pj >= kPkStages && !mbar_wait(&pk_empty[p], uint32_t(pj / kPkStages - 1) & 1u)) {
            *err = 1;
            break;
          }
          mbar_arrive_expect_tx(&pk_full[p], uint32_t(kPkBytes));
          tma_load_2d(pk + p * kPkBytes, &maps.b, c * 128, tn * kBN, &pk_full[p]);
        }
      }
      // copies still in flight (after an error) land before the CTA exits
      for (int q = pj > kPkStages ? pj - kPkStages : 0; q < pj; ++q)
        (void)mbar_wait(&pk_full[q % kPkStages], uint32_t(q / kPkStages) & 1u);
    }
  } else if (kPacked && warp >= kTcThreads / 32) {
    // decoder warps: group g = it % kTpDecGroups decodes K block it (it counts
    // this CTA's blocks).  Thread gt of the group owns 16-byte chunk c = gt % 8
    // of rows gt / 8 + 32 i of the B stage (K-major, 128-byte swizzle: chunk c
    // of row r at r * 128 + (c ^ (r % 8)) * 16; r % 8 = sw for all its rows)
    constexpr int kGT = 32 * kTpWpg;                 // threads per group
    constexpr int kPasses = 8 * kBN / kGT;           // chunks per thread and block
    const int dt = tid - kTcThreads, g = dt / kGT, gt = dt % kGT;
    // the decode table, built while the first copies are in flight: word
    // 32 b + l holds digits d0..d3 of byte b (b = sum d_k 3^k) as the int8
    // trits d_k - 1, one copy per lane l; bytes past 242 read as 121 here
    for (int wd = dt; wd < 256 * 32; wd += 32 * kTpDecWarps) {
      uint32_t x = uint32_t(wd >> 5), v = 0;
      if (x > 242u) x = 121u;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v |= ((x % 3u + 255u) & 0xFFu) << (8 * k);
        x /= 3u;
      }
      lut[wd] = v;
    }
    named_bar_sync(kTpDecBar, 32 * kTpDecWarps);
    const uint32_t c = uint32_t(gt & 7), sw = uint32_t(gt >> 3) & 7u;
    const uint32_t* lut_l = lut + lane;
    const int rem = nkb - (nch - 1) * kTcChunk;      // blocks in the last chunk
    int it = 0, pj0 = 0;
    bool ok = true;
    for (int w = blockIdx.x; w < nwork && ok && !*err; w += gridDim.x) {
      int t, j, kb0, kb1;
      work(w, t, j, kb0, kb1);
      const int c0 = kb0 / kTcChunk;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        if (it % kTpDecGroups != g) continue;
        const int pj = pj0 + kb / kTcChunk - c0, p = pj % kPkStages, sub = kb % kTcChunk;
        if (!mbar_wait(&pk_full[p], uint32_t(pj / kPkStages) & 1u)) {
          ok = false;
          break;
        }
        const int s = it % kStages;
        if (it >= kStages && !mbar_wait(&empty[s], uint32_t(it / kStages - 1) & 1u)) {
          ok = false;
          break;
        }
        // the chunk's 16 trits start at trit t0 of the packed row: packed bytes
        // b0..b0+3 hold them after al leading trits
        const uint32_t t0 = 128u * uint32_t(sub) + 16u * c;
        const uint32_t b0 = (t0 * 52429u) >> 18, al = t0 - 5u * b0;   // t0 / 5, t0 % 5
        const uint32_t w0 = b0 >> 2, w1 = w0 < 31u ? w0 + 1u : 31u;
        // the packed tile has the 128-byte swizzle too (row % 8 = sw)
        const uint32_t o0 = (((w0 >> 2) ^ sw) << 4) | ((w0 & 3u) << 2);
        const uint32_t o1 = (((w1 >> 2) ^ sw) << 4) | ((w1 & 3u) << 2);
        const uint32_t sh = 8u * (b0 & 3u), sel = 0x3210u + 0x1111u * al;
        const unsigned char* src = pk + p * kPkBytes + (gt >> 3) * 128;
        unsigned char* dst = smem + s * (kTcStageA + kTcStageB) + kTcStageA + (gt >> 3) * 128 + ((c ^ sw) << 4);
#pragma unroll
        for (int i = 0; i < kPasses; ++i) {
          const unsigned char* row = src + i * (kGT / 8) * 128;
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
          *reinterpret_cast<uint4*>(dst + i * (kGT / 8) * 128) =
              make_uint4(__byte_perm(S0, S1, sel), __byte_perm(S1, S2, sel), __byte_perm(S2, S3, sel),
                         __byte_perm(S3, S4, sel));
        }
        fence_proxy_async_smem();      // generic-proxy writes, read by the tensor cores
        __syncwarp();                  // (also: every lane's reads of the packed chunk are done)
        if (lane == 0) {
          mbar_arrive(&full[s]);
          // one arrive per block and warp; a short last chunk makes up the rest
          mbar_arrive_cnt(&pk_empty[p], kb == nkb - 1 ? uint32_t(1 + kTcChunk - rem) : 1u);
        }
      }
      pj0 += (kb1 - 1) / kTcChunk - c0 + 1;          // this item's chunks
    }
    if (!ok) *err = 1;
  } else if (warp >= 2 && warp < kTcThreads / 32) {
    // epilogue warps 2..5: warp w owns TMEM lanes 32*(w%4) .. +31
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const bool vec = kDequant ? (aligned(a.Y, 16) && (a.N & 3) == 0) : (aligned(a.acc, 16) && (a.N & 3) == 0);
    const bool pvec = (a.N & 3) == 0;                // part is 256-byte aligned
    const float beta = kDequant ? *a.beta : 0.f;
    int u = 0;
    for (int w = blockIdx.x; w < nwork; w += gridDim.x, ++u) {
      int t, j, kb0, kb1;
      work(w, t, j, kb0, kb1);
      const int b = u & 1;
      if (!mbar_wait(&acc_full[b], uint32_t(u / 2) & 1u)) {
        *err = 1;
        break;
      }
      if (*err) break;
      tc_fence_after();
      int tm, tn;
      tc_tile_coords(a, t, tm, tn);
      const int64_t m = int64_t(tm) * kTcBM + row;
      const int64_t n0 = int64_t(tn) * kBN;
      const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + uint32_t(b * kBN);
      float sbm = 0.f;
      if (kDequant && S == 1 && m < a.M) sbm = __fmul_rn(a.s[m], beta);
#pragma unroll 1
      for (int cc = 0; cc < kBN / 32; ++cc) {
        uint32_t r[32];
        tmem_ld32(taddr + uint32_t(cc * 32), r);
        tmem_ld_wait();
        const int64_t nb = n0 + cc * 32;
        if (m >= a.M || nb >= a.N) continue;
        if (S == 1) {
          tc_store32<kDequant>(a, r, m, nb, sbm, vec);
        } else {
          // this split's partial sums (tc_reduce_kernel finishes the output)
          int32_t* pr = a.part + (int64_t(j) * a.M + m) * a.N + nb;
          if (pvec && nb + 32 <= a.N) {
#pragma unroll
            for (int k = 0; k < 32; k += 4)
              *reinterpret_cast<int4*>(pr + k) = make_int4(int(r[k]), int(r[k + 1]), int(r[k + 2]), int(r[k + 3]));
          } else {
            for (int k = 0; k < 32 && nb + k < a.N; ++k) pr[k] = int(r[k]);
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

// The K-split partials [split, M, N] summed (exact int32) into acc, or through
// the epilogue's y = float32(acc) (s_m beta) [+ b_n]; four columns per thread
// when N % 4 == 0 (16-byte loads across the whole grid).
template <bool kDequant>
__global__ void __launch_bounds__(256)
tc_reduce_kernel(const int32_t* __restrict__ part, int split, int64_t M, int64_t N, const float* s,
                 const float* beta, const float* bias, float* Y, int32_t* acc) {
  griddep_wait();   // launched as a dependent of the GEMM: its partials are complete
  const bool v4 = (N & 3) == 0 && (kDequant ? aligned(Y, 16) : aligned(acc, 16));
  const int64_t per_row = v4 ? N / 4 : N;
  const int64_t total = M * per_row;
  const int64_t plane = M * N;
  const float b = kDequant ? *beta : 0.f;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t m = i / per_row, c = i - m * per_row;
    if (v4) {
      const int64_t e = m * N + 4 * c;
      int4 t = __ldcg(reinterpret_cast<const int4*>(part + e));
      for (int j = 1; j < split; ++j) {
        const int4 u = __ldcg(reinterpret_cast<const int4*>(part + j * plane + e));
        t.x = int(uint32_t(t.x) + uint32_t(u.x));
        t.y = int(uint32_t(t.y) + uint32_t(u.y));
        t.z = int(uint32_t(t.z) + uint32_t(u.z));
        t.w = int(uint32_t(t.w) + uint32_t(u.w));
      }
      if (kDequant) {
        const float sb = __fmul_rn(s[m], b);
        float4 y = make_float4(__fmul_rn(float(t.x), sb), __fmul_rn(float(t.y), sb), __fmul_rn(float(t.z), sb),
                               __fmul_rn(float(t.w), sb));
        if (bias) {
          y.x = __fadd_rn(y.x, bias[4 * c]);
          y.y = __fadd_rn(y.y, bias[4 * c + 1]);
          y.z = __fadd_rn(y.z, bias[4 * c + 2]);
          y.w = __fadd_rn(y.w, bias[4 * c + 3]);
        }
        *reinterpret_cast<float4*>(Y + e) = y;
      } else {
        *reinterpret_cast<int4*>(acc + e) = t;
      }
    } else {
      const int64_t e = m * N + c;
      uint32_t t = uint32_t(__ldcg(part + e));
      for (int j = 1; j < split; ++j) t += uint32_t(__ldcg(part + j * plane + e));
      if (kDequant) {
        float y = __fmul_rn(float(int(t)), __fmul_rn(s[m], b));
        if (bias) y = __fadd_rn(y, bias[c]);
        Y[e] = y;
      } else {
        acc[e] = int(t);
      }
    }
  }
}

// W_q from the packed format into int8 rows [N, ldq] (ldq % 16 == 0) for the
// tensor-core GEMM's TMA loads, at HBM speed: one thread per 16 packed bytes
// (80 trits), one 16-byte load and five 16-byte stores (those below ldq), so
// every warp reads 512 and writes 2560 contiguous bytes.  Trits t0..t3 of a
// byte come from a table in shared memory with one copy per lane (word
// 32 b + lane: no bank conflicts); t4 = floor(b/81) - 1 for four bytes at once
// from b * 203 in 16-bit lanes (bits 14..15, exact for b <= 242); byte_perm
// lays the 20 trits of four bytes out in order.  Row bytes from K to ldq hold
// whatever the packed padding decodes to (121: zero trits); the GEMM's tensor
// map ends at K, so it never reads them.
constexpr int kUnpackThreads = 256;

__global__ void __launch_bounds__(kUnpackThreads)
unpack5_rows_kernel(const uint8_t* __restrict__ Wp, int64_t N, int64_t ldp, int8_t* __restrict__ Wq,
                    int64_t ldq) {
  __shared__ __align__(16) uint32_t lut[256 * 32];
  static_assert(kUnpackThreads == 256, "one table row per thread");
  {
    // thread b writes the 32 lane copies of byte b's word (bytes above 242
    // are not codes: trit_word reads them as zero trits)
    const uint32_t v = trit_word(uint32_t(threadIdx.x));
    uint4* row = reinterpret_cast<uint4*>(lut + 32 * threadIdx.x);
#pragma unroll
    for (int j = 0; j < 8; ++j) row[(j + threadIdx.x) & 7] = make_uint4(v, v, v, v);
  }
  __syncthreads();
  const uint32_t* lut_l = lut + (threadIdx.x & 31);
  const int64_t cpr = ldp / 16;                 // 16-byte chunks per packed row
  const int64_t total = N * cpr;
  const bool small = total < (int64_t(1) << 32);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    int64_t row, c;
    split_index(i, cpr, small, row, c);
    const uint4 w4 = __ldg(reinterpret_cast<const uint4*>(Wp + row * ldp) + c);
    const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
    uint32_t o[20];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t four = wv[q];
      const uint32_t L0 = lut_l[(four & 0xFFu) << 5], L1 = lut_l[((four >> 8) & 0xFFu) << 5];
      const uint32_t L2 = lut_l[((four >> 16) & 0xFFu) << 5], L3 = lut_l[(four >> 24) << 5];
      const uint32_t lo = (four & 0x00FF00FFu) * 203u, hi = ((four >> 8) & 0x00FF00FFu) * 203u;
      const uint32_t T = (((__byte_perm(lo, hi, 0x7351) >> 6) & 0x03030303u) + 0x7F7F7F7Fu) ^ 0x80808080u;
      o[5 * q + 0] = L0;
      o[5 * q + 1] = __byte_perm(T, L1, 0x6540);
      o[5 * q + 2] = __byte_perm(__byte_perm(L1, T, 0x0053), L2, 0x5410);
      o[5 * q + 3] = __byte_perm(__byte_perm(L2, T, 0x0632), L3, 0x4210);
      o[5 * q + 4] = __byte_perm(L3, T, 0x7321);
    }
    int8_t* dst = Wq + row * ldq + 80 * c;
#pragma unroll
    for (int v = 0; v < 5; ++v)
      if (80 * c + 16 * v + 16 <= ldq)
        *reinterpret_cast<uint4*>(dst + 16 * v) = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
  }
}

}  // namespace bl
