// Few-row BitLinear on the tensor cores with the weights as the MMA's M side.
//
// The deployed-path contraction acc = x_q W_q^T of "ultragraph -- when the graph
// is the 1-bit LLM, part 2" (section "autograd on a byte-graph") for 5 <= M <=
// 128 token rows.  A 128-row MMA tile of X would be mostly padding here, so the
// operands swap: 128 rows of W_q are the MMA's M dimension and the M rows of X_q
// its N dimension (rounded up to 16), D^T = W_q X_q^T.  Each W element is decoded
// from its packed byte exactly once; the cost of the layer is the decode and the
// packed-weight stream, not the MMA.
//
// K blocks of 160 trits = 32 packed bytes per row, so that a thread decodes 16
// whole packed bytes (80 trits) into five 16-byte chunks, none split across
// blocks.  Per K block and stage:
//   * packed W tile [128 rows x 32 bytes] by TMA (no swizzle);
//   * X_q tile by TMA in two parts: K bytes 0..127 with the 128-byte swizzle
//     ([Np rows x 128 B]) and K bytes 128..159 with the 32-byte swizzle
//     ([Np x 32 B]);
//   * decoder warps expand the packed tile into the int8 W tile in the
//     canonical K-major "interleave" layout (no swizzle): 16-trit chunk j of row
//     r at j * 2048 + r * 16, so a warp's 32 stores of 16 bytes are contiguous.
//     Trits t0..t3 of a byte come from a table in shared memory with one copy
//     per lane (word 32 b + lane); t4 = floor(b/81) - 1 for four bytes at once
//     from b * 203 in 16-bit lanes (bits 14..15, exact for b <= 242); byte_perm
//     lays out the 20 trits of four bytes in order;
//   * five tcgen05.mma.kind::i8 (M = 128, N = Np, K = 32) into a TMEM
//     accumulator: A = W tile (interleave descriptor, chunk pair 2i, 2i+1),
//     B = X_q tile (swizzled descriptors).
// Roles: warp 0 issues the X_q loads into the stage ring, warp 22 the packed
// tiles into a ring of their own (16 deep, so 64 KB of weights are in flight per
// SM), warp 1 the MMAs, warps 2..5 drain TMEM (lane = W row, columns = X rows:
// y[m, n] for 32 consecutive n per store) with the dequant fused, warps 6..21
// decode (two groups of eight take the K blocks in turn).  With fewer 128-row
// W tiles than SMs, K is split into ranges of whole blocks whose int32
// partials [split, M, N] tc_reduce_kernel adds up (exact).  Every wait is bounded; on a timeout the kernel records kDevTimeout,
// lets copies and MMAs in flight land and frees its TMEM.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kSwBM = 128;                 // W rows per tile (MMA M)
constexpr int kSwBK = 160;                 // trits per K block (5 MMAs of K = 32)
constexpr int kSwPkBytes = kSwBM * 32;     // packed tile: 4 KB
constexpr int kSwATile = kSwBM * kSwBK;    // decoded W tile: 20 KB
constexpr int kSwMaxNp = 128;              // X rows per MMA (N), multiple of 16
constexpr int kSwMaxStages = 8;            // decoded-W / X stages (as many as fit)
constexpr int kSwPkStages = 16;            // packed tiles in flight: 64 KB per SM
constexpr int kSwDecWarps = 16, kSwDecGroups = 2;
constexpr int kSwWpg = kSwDecWarps / kSwDecGroups;
constexpr int kSwPkWarp = 6 + kSwDecWarps;             // the packed tiles' producer
constexpr int kSwThreads = 32 * (kSwPkWarp + 1);
constexpr int kSwMaxSplit = 8;
constexpr int kSwLutBytes = 256 * 128;     // word 32 b + lane
constexpr int kSwSmemMax = 232448 - 2048;  // dynamic shared memory budget

// Shared memory (from the 1024-aligned base): `nst` stages of [X128: Np x 128
// (1024-aligned) | A: 20 KB | X32: Np x 32 (256-aligned)], each rounded up to
// 1024 bytes; then the packed ring (16 x 4 KB); then the decode table.
struct SwLayout {
  int stage, nst, pk_off, lut_off, smem;
};
inline SwLayout sw_layout(int Np) {
  SwLayout l;
  l.stage = int(round_up(int64_t(Np) * 128 + kSwATile + int64_t(Np) * 32, 1024));
  const int fixed = kSwPkStages * kSwPkBytes + kSwLutBytes + 1024;
  int n = (kSwSmemMax - fixed) / l.stage;
  l.nst = n > kSwMaxStages ? kSwMaxStages : n;
  l.pk_off = l.nst * l.stage;
  l.lut_off = l.pk_off + kSwPkStages * kSwPkBytes;
  l.smem = l.lut_off + kSwLutBytes + 1024;
  return l;
}

struct alignas(64) SwMaps {
  CUtensorMap x128;   // X_q [M, ldx] int8, boxes {128, Np}, 128-byte swizzle
  CUtensorMap x32;    // X_q [M, ldx] int8, boxes {32, Np}, 32-byte swizzle
  CUtensorMap wp;     // packed W [N, ldp] uint8, boxes {32, 128}, no swizzle
};

struct SwArgs {
  int64_t M, N, K;
  int Np;              // MMA N: round_up(M, 16)
  const float* s;      // row scales, or nullptr (integer product)
  const float* beta;
  const float* bias;
  float* Y;            // [M, N] float32, or nullptr
  int32_t* acc;        // [M, N] int32 when Y is nullptr
  int tiles, split;
  int32_t* part;       // [split, M, N] int32 (split > 1)
  int nst, stage, pk_off, lut_off;   // shared-memory layout (sw_layout)
};

// The table of trits t0..t3 per byte (word 32 b + lane), a compile-time constant.
struct TritLut128 {
  uint32_t w[256 * 32];
};
constexpr TritLut128 make_trit_lut128() {
  TritLut128 t{};
  for (uint32_t b = 0; b < 256; ++b) {
    uint32_t x = b > 242u ? 121u : b, v = 0;
    for (int k = 0; k < 4; ++k) {
      v |= ((x % 3u + 255u) & 0xFFu) << (8 * k);
      x /= 3u;
    }
    for (uint32_t l = 0; l < 32; ++l) t.w[b * 32 + l] = v;
  }
  return t;
}
__device__ __align__(128) const TritLut128 g_trit_lut128 = make_trit_lut128();

// Shared-memory descriptors: K-major, no swizzle (core matrices of 8 rows x 16
// bytes; LBO = K-direction stride, SBO = row-group stride) and K-major with the
// 32-byte swizzle (rows of 32 bytes, 8-row groups 256 bytes apart).
__device__ __forceinline__ uint64_t umma_desc_k_interleave(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((addr & 0x3FFFFu) >> 4);
  d |= uint64_t((lbo >> 4) & 0x3FFFu) << 16;
  d |= uint64_t((sbo >> 4) & 0x3FFFu) << 32;
  d |= uint64_t(1) << 46;
  return d;   // layout type 0: no swizzle
}
__device__ __forceinline__ uint64_t umma_desc_k_sw32(uint32_t addr) {
  uint64_t d = 0;
  d |= uint64_t((addr & 0x3FFFFu) >> 4);
  d |= uint64_t(1) << 16;
  d |= uint64_t(256 >> 4) << 32;
  d |= uint64_t(1) << 46;
  d |= uint64_t(6) << 61;     // SWIZZLE_32B
  return d;
}

// The TMEM load of 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

template <bool kDequant>
__global__ void __launch_bounds__(kSwThreads, 1)
gemm_swap_kernel(const __grid_constant__ SwMaps maps, const SwArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t ld_full[kSwMaxStages], dec_full[kSwMaxStages], empty[kSwMaxStages];
  __shared__ uint64_t pk_full[kSwPkStages], pk_empty[kSwPkStages];
  __shared__ uint64_t acc_full[2], acc_empty[2], drain, lut_bar;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* err = &s_err;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  uint32_t* lut = reinterpret_cast<uint32_t*>(smem + a.lut_off);
  const int Np = a.Np, nst = a.nst;
  const int nkb = int(ceil_div(a.K, kSwBK));
  const int S = a.split;
  const int nwork = a.tiles * S;
  auto work = [&](int w, int& t, int& kb0, int& kb1, int& j) {
    t = w / S;
    j = w - t * S;
    kb0 = j * nkb / S;
    kb1 = (j + 1) * nkb / S;
  };
  auto stage_x128 = [&](int s) { return smem + s * a.stage; };
  auto stage_a = [&](int s) { return smem + s * a.stage + Np * 128; };
  auto stage_x32 = [&](int s) { return smem + s * a.stage + Np * 128 + kSwATile; };
  auto stage_pk = [&](int p) { return smem + a.pk_off + p * kSwPkBytes; };
  const uint32_t x_bytes = uint32_t(Np) * uint32_t(kSwBK);

  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < nst; ++s) {
      mbar_init(&ld_full[s], 1);
      mbar_init(&dec_full[s], kSwWpg);
      mbar_init(&empty[s], 1);
    }
    for (int p = 0; p < kSwPkStages; ++p) {
      mbar_init(&pk_full[p], 1);
      mbar_init(&pk_empty[p], kSwWpg);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(&drain, 1);
    mbar_init(&lut_bar, 1);
    fence_mbar_init();
    prefetch_tmap(&maps.x128);
    prefetch_tmap(&maps.x32);
    prefetch_tmap(&maps.wp);
    mbar_arrive_expect_tx(&lut_bar, kSwLutBytes);
    bulk_g2s(lut, &g_trit_lut128, kSwLutBytes, &lut_bar);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 256);
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
        int t, kb0, kb1, j;
        work(w, t, kb0, kb1, j);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % nst;
          if (it >= nst && !mbar_wait(&empty[s], uint32_t(it / nst - 1) & 1u)) {
            *err = 1;
            break;
          }
          mbar_arrive_expect_tx(&ld_full[s], x_bytes);
          tma_load_2d(stage_x128(s), &maps.x128, kb * kSwBK, 0, &ld_full[s]);
          tma_load_2d(stage_x32(s), &maps.x32, kb * kSwBK + 128, 0, &ld_full[s]);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_i8(kSwBM, Np);
      int it = 0, u = 0;
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x, ++u) {
        int t, kb0, kb1, j;
        work(w, t, kb0, kb1, j);
        const int b = u & 1;
        if (u >= 2 && !mbar_wait(&acc_empty[b], uint32_t(u / 2 - 1) & 1u)) {
          *err = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem + uint32_t(b * kSwMaxNp);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % nst;
          if (!mbar_wait(&ld_full[s], uint32_t(it / nst) & 1u) ||
              !mbar_wait(&dec_full[s], uint32_t(it / nst) & 1u)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t xa = smem_u32(stage_x128(s)), x32 = smem_u32(stage_x32(s)), wa = smem_u32(stage_a(s));
#pragma unroll
          for (int i = 0; i < 5; ++i) {
            const uint64_t adesc = umma_desc_k_interleave(wa + uint32_t(i) * 4096u, 2048u, 128u);
            const uint64_t bdesc = i < 4 ? umma_desc_k_sw128(xa + 32u * uint32_t(i)) : umma_desc_k_sw32(x32);
            umma_i8(d, adesc, bdesc, idesc, (kb > kb0 || i > 0) ? 1u : 0u);
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
  } else if (warp >= 6 && warp < kSwPkWarp) {
    // decoder warps: group g decodes the blocks it % 2 == g; thread gt of the
    // group owns row gt / 2 and packed bytes 16 (gt % 2) .. +15 of the block
    constexpr int kGT = 32 * kSwWpg;                 // 256 threads: 128 rows x 2 halves
    const int dt = tid - 192, g = dt / kGT, gt = dt % kGT;
    const int r = gt >> 1, h = gt & 1;
    const uint32_t* lut_l = lut + lane;
    bool ok = mbar_wait(&lut_bar, 0u);
    int it = 0;
    for (int w = blockIdx.x; w < nwork && ok && !*err; w += gridDim.x) {
      int t, kb0, kb1, j;
      work(w, t, kb0, kb1, j);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        if (it % kSwDecGroups != g) continue;
        const int s = it % nst, pp = it % kSwPkStages;
        if (!mbar_wait(&pk_full[pp], uint32_t(it / kSwPkStages) & 1u) ||
            !mbar_wait(&ld_full[s], uint32_t(it / nst) & 1u)) {
          ok = false;
          break;
        }
        const uint4 p = *reinterpret_cast<const uint4*>(stage_pk(pp) + r * 32 + h * 16);
        const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
        uint32_t o[20];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t four = pw[q];
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
        unsigned char* dst = stage_a(s) + (5 * h) * 2048 + r * 16;
#pragma unroll
        for (int v = 0; v < 5; ++v)
          *reinterpret_cast<uint4*>(dst + v * 2048) = make_uint4(o[4 * v], o[4 * v + 1], o[4 * v + 2], o[4 * v + 3]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&dec_full[s]);
          mbar_arrive(&pk_empty[pp]);
        }
      }
    }
    if (!ok) *err = 1;
  } else if (warp == kSwPkWarp) {
    // packed producer: up to 16 packed tiles ahead of the decoders
    if (lane == 0) {
      int it = 0;
      for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x) {
        int t, kb0, kb1, j;
        work(w, t, kb0, kb1, j);
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int pp = it % kSwPkStages;
          if (it >= kSwPkStages && !mbar_wait(&pk_empty[pp], uint32_t(it / kSwPkStages - 1) & 1u)) {
            *err = 1;
            break;
          }
          mbar_arrive_expect_tx(&pk_full[pp], uint32_t(kSwPkBytes));
          tma_load_2d(stage_pk(pp), &maps.wp, kb * 32, t * kSwBM, &pk_full[pp]);
        }
      }
      // copies still in flight (after an error) land before the CTA exits
      for (int q = it > kSwPkStages ? it - kSwPkStages : 0; q < it; ++q)
        (void)mbar_wait(&pk_full[q % kSwPkStages], uint32_t(q / kSwPkStages) & 1u);
    }
  } else if (warp >= 2 && warp < 6) {
    // epilogue warps 2..5: TMEM lane = W row of the tile, columns = X rows
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    const float beta = kDequant ? *a.beta : 0.f;
    int u = 0;
    for (int w = blockIdx.x; w < nwork; w += gridDim.x, ++u) {
      int t, kb0, kb1, j;
      work(w, t, kb0, kb1, j);
      const int b = u & 1;
      if (!mbar_wait(&acc_full[b], uint32_t(u / 2) & 1u)) {
        *err = 1;
        break;
      }
      if (*err) break;
      tc_fence_after();
      const int64_t n = int64_t(t) * kSwBM + rl;
      const uint32_t taddr = tmem + (uint32_t(q * 32) << 16) + uint32_t(b * kSwMaxNp);
      const float bn = (kDequant && a.bias && n < a.N) ? a.bias[n] : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < Np; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(taddr + uint32_t(c0), v);
        tmem_ld_wait();
        if (n >= a.N) continue;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int64_t m = c0 + c;
          if (m >= a.M) break;
          if (S > 1) {
            a.part[(int64_t(j) * a.M + m) * a.N + n] = int(v[c]);
          } else if (kDequant) {
            float y = __fmul_rn(float(int(v[c])), __fmul_rn(a.s[m], beta));
            if (a.bias) y = __fadd_rn(y, bn);
            a.Y[m * a.N + n] = y;
          } else {
            a.acc[m * a.N + n] = int(v[c]);
          }
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
    tmem_dealloc(tmem, 256);
  }
  if (tid == 0) (void)mbar_wait(&lut_bar, 0u);   // the table copy has landed before the CTA exits
}

}  // namespace bl
