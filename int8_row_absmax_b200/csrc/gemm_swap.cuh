// Few-row BitLinear on the tensor cores with the weights as the MMA's M side.
//
// The deployed-path contraction acc = x_q W_q^T of "ultragraph -- when the graph
// is the 1-bit LLM, part 2" (section "autograd on a byte-graph") for 1 <= M <=
// 128 token rows.  A 128-row MMA tile of X would be mostly padding here, so the
// operands swap: 128 rows of W_q are the MMA's M dimension and the M rows of X_q
// its N dimension (rounded up to 16), D^T = W_q X_q^T.  Each W element is decoded
// from its packed byte exactly once; the cost of the layer is the decode and the
// packed-weight stream, not the MMA.
//
// K blocks of 160 trits = 32 packed bytes per row.  The decoded W tile never
// touches shared memory: each decoder thread owns one W row (one TMEM lane),
// expands its 32 packed bytes into 40 words of int8 trits and stores them into
// tensor memory (tcgen05.st), from where the MMA reads its A operand.  The
// words come in the decode order of trit_table.cuh (t0..t3 of each byte from
// the per-lane table, then t4 of four bytes at once), and X_q arrives in the
// same order, written so by the activation quantizer: no byte is shuffled.
// Work goes in chunks of four K blocks (640 trits, 128 packed bytes per row):
//   * packed W: one TMA box of [128 rows x 128 bytes] per chunk (128-byte
//     swizzle), a ring of four, so 64 KB of weights are in flight per SM;
//   * X_q: one 3-D TMA box per chunk, the chunk's 640 code bytes of the Np rows
//     as five 128-byte swizzle atoms ([5][Np][128 B]), in a ring of as many
//     chunks as fit (for few rows, a CTA's whole K range), so the X loads are
//     few, large and issued far ahead of the MMAs that read them;
//   * decoders: four groups of four warps (one warp per TMEM lane quarter), the
//     group g decoding block g of every chunk; 40 TMEM columns per block;
//   * per block, five tcgen05.mma.kind::i8 (M = 128, N = Np, K = 32): A from
//     TMEM columns 8i.., B at position 160 h + 32 i of the chunk (atom and
//     offset of the 128-byte swizzle).
// Roles: warp 0 issues the X_q loads, warp 22 the packed boxes, warp 1 holds
// the TMEM allocation, warps 6..21 decode, warps 2..5 issue the MMAs (one
// thread issues a tcgen05.mma only every 60-110 ns, and issuers in several
// warps overlap) into an accumulator each, then drain TMEM (lane = W row,
// columns = X rows), add the accumulators and fuse the dequant into the
// stores.  With fewer 128-row W tiles than SMs, K is split into ranges of
// whole chunks whose int32 partials [split, M, N] tc_reduce_kernel adds up
// (exact).  The launch is a programmatic dependent one: barriers, TMEM, the
// decode table (written into shared memory by the CTA) and (for static
// weights) the first packed boxes are set up while the previous kernel
// finishes.  Every wait is bounded; on a timeout the kernel records
// kDevTimeout, lets copies and MMAs in flight land and frees its TMEM.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "trit_table.cuh"

namespace bl {

constexpr int kSwBM = 128;                 // W rows per tile (MMA M)
constexpr int kSwBK = 160;                 // trits per K block (5 MMAs of K = 32)
constexpr int kSwBoxKb = 4;                // K blocks per packed box (128 bytes of a row)
constexpr int kSwBoxBytes = kSwBM * 128;   // packed box: 16 KB
constexpr int kSwPkSlots = 4;              // packed boxes in flight: 64 KB per SM
constexpr int kSwMaxNp = 128;              // X rows per MMA (N), multiple of 16
constexpr int kSwChunkX = 5 * 128;         // X_q bytes per row and chunk (640 trits)
constexpr int kSwMaxXStages = 16;          // X chunks in flight (as many as fit)
constexpr int kSwMaxAStages = 8;           // decoded W blocks in flight (TMEM), as many as fit
constexpr int kSwAccCols = 256;            // at most 256 TMEM columns of accumulators (one per MMA issuer)
constexpr int kSwAStride = 64;             // TMEM columns per A stage (40 used), 64-column aligned
constexpr int kSwTmemCols = 512;
constexpr int kSwDecGroups = 4, kSwDecWarps = 4 * kSwDecGroups;
constexpr int kSwPkWarp = 6 + kSwDecWarps;             // the packed boxes' producer
constexpr int kSwThreads = 32 * (kSwPkWarp + 1);
constexpr int kSwMaxSplit = 8;
constexpr int kSwSmemMax = 232448 - 1024;  // dynamic shared memory budget

static_assert(kSwAccCols + 4 * kSwAStride <= kSwTmemCols, "TMEM columns");

// Shared memory (from the 1024-aligned base): the packed ring (4 x 16 KB), the
// decode table (64 KB), then `nst` X chunks of [5 atoms][Np rows][128 B].  X has
// a ring of its own, deeper than the four TMEM stages of decoded W: its loads
// (from L2) are issued far ahead and never wait for an MMA just issued.
struct SwLayout {
  int xst, nst, lut_off, x_off, smem;
};
inline SwLayout sw_layout(int Np) {
  SwLayout l;
  l.xst = int(round_up(int64_t(Np) * kSwChunkX, 1024));
  l.lut_off = kSwPkSlots * kSwBoxBytes;
  l.x_off = l.lut_off + int(kLutBytes);
  int n = (kSwSmemMax - 1024 - l.x_off) / l.xst;
  l.nst = n > kSwMaxXStages ? kSwMaxXStages : n;
  l.smem = l.x_off + l.nst * l.xst + 1024;
  return l;
}

// MMA issuers: four while four accumulators of Np columns fit in the 256
// accumulator columns of TMEM, else two (a divisor of the four A stages, so
// that every stage is always released by the same issuer, in order).
inline int sw_mma_warps(int Np) { return Np <= kSwAccCols / 4 ? 4 : 2; }
// TMEM: the accumulators (issuers x Np columns) from column 0, then the A
// stages from the next multiple of 64 columns, as many as fit (up to 8), so
// that a decoder group fills its next stage while the MMAs read the last one.
inline int sw_a_col0(int Np) { return int(round_up(int64_t(sw_mma_warps(Np)) * Np, kSwAStride)); }
inline int sw_a_stages(int Np) {
  const int n = (kSwTmemCols - sw_a_col0(Np)) / kSwAStride;
  return n > kSwMaxAStages ? kSwMaxAStages : n;
}

struct alignas(64) SwMaps {
  CUtensorMap x;      // X_q in decode order as {128 B, M rows, ldx/128 atoms}, boxes {128, Np, 5}, 128-byte swizzle
  CUtensorMap wp;     // packed W [N, ldp] uint8, boxes {128, 128}, 128-byte swizzle
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
  int nst, xst, lut_off, x_off;   // shared-memory layout (sw_layout); nst X stages
  int static_w;        // 1: W is not written by earlier kernels (copied before the dependency wait)
  int mma_warps;       // MMA issuers, one accumulator each (sw_mma_warps)
  int a_col0, nsa;     // TMEM column of the first A stage, number of A stages
};

// The TMEM load of 16 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// 40 words of int8 trits (decode order) of the 32 packed bytes p0 | p1 of a row.
__device__ __forceinline__ void sw_decode_block(const unsigned char* lut, uint32_t lanebase, const uint4& p0,
                                                const uint4& p1, uint32_t* o) {
  const uint32_t pw[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const uint32_t w = pw[q];
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) o[5 * q + bb] = lut_t0123(lut, w, lanebase, bb);
    o[5 * q + 4] = t4_word(w);
  }
}

template <bool kDequant>
__global__ void __launch_bounds__(kSwThreads, 1)
gemm_swap_kernel(const __grid_constant__ SwMaps maps, const SwArgs a) {
  extern __shared__ unsigned char smem_raw[];
  __shared__ uint64_t ld_full[kSwMaxXStages], x_empty[kSwMaxXStages], dec_full[kSwMaxAStages], a_empty[kSwMaxAStages];
  __shared__ uint64_t pk_full[kSwPkSlots], pk_empty[kSwPkSlots];
  __shared__ uint64_t acc_full, acc_empty, drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_err;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  volatile int* err = &s_err;
  const uint32_t base = (smem_u32(smem_raw) + 1023u) & ~1023u;
  unsigned char* smem = smem_raw + (base - smem_u32(smem_raw));
  const unsigned char* lut = smem + a.lut_off;
  const int Np = a.Np, nst = a.nst, nsa = a.nsa;
  const int nkb = int(ceil_div(a.K, kSwBK));
  const int nch = (nkb + kSwBoxKb - 1) / kSwBoxKb;   // chunks of four K blocks
  const int S = a.split;
  const int nwork = a.tiles * S;
  // work item w: W tile t, K split j = chunks c0..c1 = blocks kb0..kb1
  auto work = [&](int w, int& t, int& kb0, int& kb1, int& j) {
    t = w / S;
    j = w - t * S;
    kb0 = kSwBoxKb * (j * nch / S);
    kb1 = min(nkb, kSwBoxKb * ((j + 1) * nch / S));
  };
  auto stage_x = [&](int s) { return smem + a.x_off + s * a.xst; };
  auto box = [&](int slot) { return smem + slot * kSwBoxBytes; };
  const uint32_t x_bytes = uint32_t(Np) * uint32_t(kSwChunkX);

  // ---- prologue: nothing here reads what an earlier kernel may still write
  if (tid == 0) {
    s_err = 0;
    for (int s = 0; s < nst; ++s) {
      mbar_init(&ld_full[s], 1);
      mbar_init(&x_empty[s], a.mma_warps);  // every issuer, once per chunk
    }
    for (int s = 0; s < a.nsa; ++s) {
      mbar_init(&dec_full[s], 4);            // the four warps of a decoder group
      mbar_init(&a_empty[s], 1);
    }
    for (int p = 0; p < kSwPkSlots; ++p) {
      mbar_init(&pk_full[p], 1);
      mbar_init(&pk_empty[p], kSwDecWarps);  // every decoder warp, once per box
    }
    mbar_init(&acc_full, a.mma_warps);
    mbar_init(&acc_empty, 4);
    mbar_init(&drain, a.mma_warps);
    fence_mbar_init();
    prefetch_tmap(&maps.x);
    prefetch_tmap(&maps.wp);
  }
  build_trit_lut(smem + a.lut_off, tid, kSwThreads);   // visible after the barrier below
  if (warp == 1) {
    tmem_alloc(&s_tmem, kSwTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // The single-issuer roles (X loads, packed loads, MMAs) run on whole warps:
  // all 32 lanes take the loop and the waits, lane 0 issues.  A lane looping
  // alone while the rest of its warp waits at the final barrier was measured to
  // cost a few hundred nanoseconds per iteration.
  if (warp == 0) {
    // X_q chunks: written by the previous kernel (the activation quantizer)
    griddep_wait();
    griddep_launch_dependents();
    int it = 0;              // chunks issued
    for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x) {
      int t, kb0, kb1, j;
      work(w, t, kb0, kb1, j);
      bool ok = true;
      for (int c = kb0 / kSwBoxKb; c * kSwBoxKb < kb1; ++c, ++it) {
        const int s = it % nst;
        if (it >= nst && !__all_sync(0xffffffffu, mbar_wait(&x_empty[s], uint32_t(it / nst - 1) & 1u))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&ld_full[s], x_bytes);
          tma_load_3d(stage_x(s), &maps.x, 0, 0, 5 * c, &ld_full[s]);
        }
        __syncwarp();
      }
      if (!ok) {
        *err = 1;
        break;
      }
    }
    // copies still in flight (after an error) land before the CTA exits
    for (int q = it > nst ? it - nst : 0; q < it; ++q) (void)mbar_wait(&ld_full[q % nst], uint32_t(q / nst) & 1u);
  } else if (warp == kSwPkWarp) {
    // packed boxes: four K blocks of 128 W rows each
    if (!a.static_w) griddep_wait();
    int bi = 0;
    for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x) {
      int t, kb0, kb1, j;
      work(w, t, kb0, kb1, j);
      const int nbox = (kb1 - kb0 + kSwBoxKb - 1) / kSwBoxKb;
      bool ok = true;
      for (int b = 0; b < nbox; ++b, ++bi) {
        const int slot = bi % kSwPkSlots;
        if (bi >= kSwPkSlots &&
            !__all_sync(0xffffffffu, mbar_wait(&pk_empty[slot], uint32_t(bi / kSwPkSlots - 1) & 1u))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&pk_full[slot], uint32_t(kSwBoxBytes));
          tma_load_2d(box(slot), &maps.wp, (kb0 + kSwBoxKb * b) * 32, t * kSwBM, &pk_full[slot]);
        }
        __syncwarp();
      }
      if (!ok) {
        *err = 1;
        break;
      }
    }
    for (int q = bi > kSwPkSlots ? bi - kSwPkSlots : 0; q < bi; ++q)
      (void)mbar_wait(&pk_full[q % kSwPkSlots], uint32_t(q / kSwPkSlots) & 1u);
  } else if (warp >= 6 && warp < kSwPkWarp) {
    // decoders: group g (four warps, one per TMEM lane quarter) decodes block
    // 4b + g of every box b; thread = W row r of the tile = TMEM lane r
    const int g = (warp - 6) >> 2, qd = warp & 3;
    const int r = qd * 32 + lane;
    const uint32_t lanebase = uint32_t(lane) * 4u;
    const uint32_t tlane = tmem + (uint32_t(qd * 32) << 16);
    // 16-byte chunks 2g, 2g + 1 of the row's 128 bytes, at their swizzled places
    const int c0 = (2 * g) ^ (r & 7), c1 = (2 * g + 1) ^ (r & 7);
    bool ok = true;
    int it = 0, bi = 0;
    for (int w = blockIdx.x; w < nwork && ok && !*err; w += gridDim.x) {
      int t, kb0, kb1, j;
      work(w, t, kb0, kb1, j);
      const int nl = kb1 - kb0;
      const int nbox = (nl + kSwBoxKb - 1) / kSwBoxKb;
      for (int b = 0; b < nbox; ++b, ++bi) {
        const int slot = bi % kSwPkSlots;
        if (!__all_sync(0xffffffffu, mbar_wait(&pk_full[slot], uint32_t(bi / kSwPkSlots) & 1u))) {
          ok = false;
          break;
        }
        const int l = kSwBoxKb * b + g;
        if (l < nl) {
          const int itb = it + l, s = itb % nsa;
          if (itb >= nsa && !__all_sync(0xffffffffu, mbar_wait(&a_empty[s], uint32_t(itb / nsa - 1) & 1u))) {
            ok = false;
            break;
          }
          const unsigned char* rowp = box(slot) + r * 128;
          const uint4 p0 = *reinterpret_cast<const uint4*>(rowp + 16 * c0);
          const uint4 p1 = *reinterpret_cast<const uint4*>(rowp + 16 * c1);
          uint32_t o[40];
          sw_decode_block(lut, lanebase, p0, p1, o);
          tc_fence_after();            // the MMAs that read this stage before are complete
          const uint32_t ta = tlane + uint32_t(a.a_col0 + s * kSwAStride);
          tmem_st32(ta, o);
          tmem_st8(ta + 32u, o + 32);
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&dec_full[s]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&pk_empty[slot]);
      }
      it += nl;
    }
    if (!ok) *err = 1;
  } else if (warp >= 2 && warp < 6) {
    // warps 2..5: MMA issuers, then the epilogue.  Issuer m (< nmw) takes the
    // blocks m, m + nmw, ... of every chunk into an accumulator of its own
    // (TMEM columns m Np ..): one thread issues an MMA every 60-110 ns, and
    // issuers in several warps overlap on the tensor core.  Then TMEM lane =
    // W row of the tile, columns = X rows: the accumulators are added (exact
    // int32) and the dequant is fused into the stores.
    const int mw = warp - 2, nmw = a.mma_warps;
    const int q = warp & 3;
    const int rl = q * 32 + lane;
    const uint32_t idesc = umma_idesc_i8(kSwBM, Np);
    griddep_wait();                    // s, beta, bias come from earlier kernels; Y may be read by them
    const float beta = kDequant ? *a.beta : 0.f;
    int it = 0, u = 0, ci = 0;         // blocks, work items, X chunks consumed
    for (int w = blockIdx.x; w < nwork && !*err; w += gridDim.x, ++u) {
      int t, kb0, kb1, j;
      work(w, t, kb0, kb1, j);
      const int nl = kb1 - kb0;
      if (u >= 1 && !__all_sync(0xffffffffu, mbar_wait(&acc_empty, uint32_t(u - 1) & 1u))) {   // drained
        *err = 1;
        break;
      }
      tc_fence_after();
      bool ok = true;
      if (mw < nmw) {
        const uint32_t dacc = tmem + uint32_t(mw * Np);
        bool first = true;
        for (int l0 = 0; l0 < nl && ok; l0 += kSwBoxKb, ++ci) {     // chunk ci
          const int s = ci % nst;
          const int hend = min(kSwBoxKb, nl - l0);
          for (int h = mw; h < hend; h += nmw) {
            const int itb = it + l0 + h, sa = itb % nsa;
            const bool got = mbar_wait(&ld_full[s], uint32_t(ci / nst) & 1u) &&
                             mbar_wait(&dec_full[sa], uint32_t(itb / nsa) & 1u);
            if (!__all_sync(0xffffffffu, got)) {
              ok = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint32_t xa = smem_u32(stage_x(s));
              const uint32_t acol = tmem + uint32_t(a.a_col0 + sa * kSwAStride);
#pragma unroll
              for (int i = 0; i < 5; ++i) {
                const uint32_t pos = uint32_t(kSwBK * h + 32 * i);   // position in the chunk
                const uint64_t bdesc = umma_desc_k_sw128(xa + (pos >> 7) * uint32_t(Np * 128) + (pos & 127u));
                umma_i8_ts(dacc, acol + 8u * uint32_t(i), bdesc, idesc, (first && i == 0) ? 0u : 1u);
              }
              umma_commit(&a_empty[sa]);
            }
            first = false;
            __syncwarp();
          }
          if (lane == 0) umma_commit(&x_empty[s]);   // this issuer is done with the chunk
          __syncwarp();
        }
        if (lane == 0) umma_commit(&acc_full);
        __syncwarp();
      } else {
        ci += (nl + kSwBoxKb - 1) / kSwBoxKb;
      }
      it += nl;
      if (!ok) {
        *err = 1;
        break;
      }
      // epilogue: the nmw accumulators that this item wrote (issuers with a block)
      if (!__all_sync(0xffffffffu, mbar_wait(&acc_full, uint32_t(u) & 1u))) {
        *err = 1;
        break;
      }
      if (*err) break;
      tc_fence_after();
      const int64_t n = int64_t(t) * kSwBM + rl;
      const uint32_t taddr = tmem + (uint32_t(q * 32) << 16);
      const float bn = (kDequant && a.bias && n < a.N) ? a.bias[n] : 0.f;
      const int nacc = min(nmw, nl);
#pragma unroll 1
      for (int c0 = 0; c0 < Np; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(taddr + uint32_t(c0), v);
        for (int c1 = 1; c1 < nacc; c1 += 2) {           // the other accumulators, two loads in flight
          uint32_t w0[16], w1[16];
          tmem_ld16(taddr + uint32_t(c1 * Np + c0), w0);
          if (c1 + 1 < nacc) tmem_ld16(taddr + uint32_t((c1 + 1) * Np + c0), w1);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 16; ++c) v[c] += w0[c] + (c1 + 1 < nacc ? w1[c] : 0u);
        }
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
      if (lane == 0) mbar_arrive(&acc_empty);
    }
    if (mw < nmw && lane == 0) umma_commit(&drain);   // every MMA of this issuer has completed
    __syncwarp();
  }

  __syncthreads();
  if (warp == 1) {
    const bool drained = mbar_wait(&drain, 0u);
    if ((!drained || *err) && lane == 0) raise_status(kDevTimeout);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kSwTmemCols);
  }
}

}  // namespace bl
