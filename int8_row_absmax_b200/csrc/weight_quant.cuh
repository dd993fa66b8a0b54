// Absmean ternarization of a weight tensor.
//
// "ultragraph -- when the graph is the 1-bit LLM, part 2", section "the bytes":
//   beta = (1/n) sum_i |W_i| + eps,   W_q = clip(round(W / beta), -1, 1).
//
// beta needs the exact sum of n float32 magnitudes: any float32 or float64 running
// sum depends on the reduction order, and a one-ulp change in beta flips codes
// that sit on a rounding boundary.  Every finite float32 |w| is m * 2^(e-150)
// (m < 2^24, e the biased exponent), so the sum is an integer in units of 2^-149.
//
//   absmean (one launch, one persistent CTA per SM):
//     0. the weights stream through a ring of shared-memory stages filled by
//        32 KB bulk copies (TMA engine) that one producer warp issues; chunks
//        are handed out dynamically from a counter in the workspace, so SMs
//        that get their bytes sooner take more chunks instead of waiting for
//        the slowest one; 16 consumer warps read the stages (full / empty
//        mbarrier pair per stage, bounded waits);
//     1. each thread adds magnitudes with exponents in a fast window [110, 141]
//        into a 96-bit fixed-point accumulator (unit 2^-40): one mad.wide.u32 per
//        weight adds m * 2^(e-110), where shl.b32 turns any shift outside the
//        window into a zero factor; a warp-uniform slow path (taken only for a
//        batch that holds such a weight) puts those magnitudes into
//        per-exponent 64-bit bins in shared memory;
//     2. each CTA adds its three 32-bit limb sums and its non-zero bins into the
//        workspace accumulator block with 64-bit atomics (integer adds are exact,
//        so the total does not depend on the schedule), then takes a ticket;
//     3. the CTA that takes the last ticket rounds the exact total once to
//        float64 (nearest-even): when no exponent bin was used the total is the
//        96-bit fixed-point sum, converted by one correctly rounded
//        integer-to-double (a sticky bit stands for any dropped low bits);
//        otherwise every bin and limb is placed at its bit offset in a 512-bit
//        integer (word-parallel, then one carry pass) and rounded from there.
//        Then it divides by n in float64 (IEEE), rounds to float32, adds eps in
//        float32, and clears the block again.
//     The block must therefore be zero before the first call on a workspace;
//     every call leaves it zero.  A magic word that must read 0 catches most
//     workspaces that were never cleared (reported as BL_ERR_WORKSPACE).
//   ternarize*:       round(w/beta) != 0 exactly when float32(|w|/beta) > 0.5,
//                     i.e. (ties go to the even 0.5) when the real quotient exceeds
//                     0.5 + 2^-25.  So the code is nonzero iff |w| > beta (0.5 +
//                     2^-25); that product is exact in float64, and T = the least
//                     float32 above it turns the test into one float compare per
//                     weight, with the same codes as the IEEE division.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kAbsConsumers = 512;                          // 16 consumer warps
constexpr int kAbsThreads = kAbsConsumers + 32;             // + 1 producer warp
constexpr int kAbsChunkFloats = 8192;                       // 32 KB per bulk copy
constexpr uint32_t kAbsChunkBytes = kAbsChunkFloats * 4;
constexpr int kAbsStages = 6;                               // 192 KB in flight per SM
constexpr int kAbsSmem = kAbsStages * int(kAbsChunkBytes);
constexpr uint32_t kFastLo = 110;  // exponent whose mantissa LSB is 2^-40
constexpr uint32_t kFastHi = 141;  // m * 2^31 < 2^55: a batch of 16 stays below 2^59

// Accumulator block at the start of the weight-quantization workspace.
constexpr int kAbsMaxCtas = 256;
struct AbsAccum {
  unsigned long long bins[256]; // sum of m per biased exponent outside the window
  unsigned int ticket;          // CTAs done so far in the current call
  unsigned int magic;           // must be 0: a never-cleared workspace reads non-zero
  unsigned int next_chunk;      // next 32 KB chunk of W to hand out
  unsigned int pad_;
  unsigned long long slot[kAbsMaxCtas][4];  // per-CTA sums of the three 32-bit limbs
  // single-pass quantization (weight_fused.cuh): the fix-up mode chosen by the
  // last CTA, the fall-back flags, the two grid barriers and the exit count (all
  // zero between calls), and each CTA's sums of sampled run means
  unsigned int mode;
  unsigned int overflow;
  unsigned int bar_a;
  unsigned int flag_b;
  unsigned int exit_cnt;
  unsigned int bins_used;
  unsigned long long tot[3];        // exact pass: the three 32-bit limb sums over all CTAs
  double dsum;                      // float64 sum of |w| over all CTAs
  unsigned int ticket2;             // exact pass: CTAs done
  unsigned int flag_c;              // exact pass: beta published
  unsigned int exit2;               // forward: CTAs done writing Y
  unsigned int pad4_;
  double est_part[kAbsMaxCtas][2];  // per CTA: sampled chunk mean (-1: none) and its square
};
constexpr size_t kAbsWsBytes = 16384;
static_assert(sizeof(AbsAccum) <= kAbsWsBytes, "accumulator block");

// 1 << s for s < 32, and 0 for any larger (unsigned) s: PTX clamps the shift.
__device__ __forceinline__ uint32_t shl_clamp(uint32_t x, uint32_t sft) {
  uint32_t r;
  asm("shl.b32 %0, %1, %2;" : "=r"(r) : "r"(x), "r"(sft));
  return r;
}

__device__ __forceinline__ unsigned long long mad_wide_u32(uint32_t a, uint32_t b,
                                                           unsigned long long c) {
  unsigned long long d;
  asm("mad.wide.u32 %0, %1, %2, %3;" : "=l"(d) : "r"(a), "r"(b), "l"(c));
  return d;
}

// Fast path for one weight: m * 2^(e-110) if e is in the window, else 0;
// `out` records a nonzero weight outside the window.
__device__ __forceinline__ unsigned long long absmean_fast(float w, unsigned long long acc,
                                                           bool& out) {
  const uint32_t u = __float_as_uint(w) & 0x7FFFFFFFu;
  const uint32_t sh = (u >> 23) - kFastLo;  // wraps for e < kFastLo
  out |= sh > (kFastHi - kFastLo);
  return mad_wide_u32((u & 0x7FFFFFu) | 0x800000u, shl_clamp(1u, sh), acc);
}

// Slow path for one weight outside the fast window [lo_e, lo_e + 31] (zero adds
// nothing).
__device__ __forceinline__ void absmean_slow(float w, unsigned long long* s_bins, bool& bad,
                                             uint32_t lo_e = kFastLo) {
  const uint32_t u = __float_as_uint(w) & 0x7FFFFFFFu;
  const uint32_t e = u >> 23;
  if (e - lo_e <= kFastHi - kFastLo) return;  // counted by the fast path
  if (e == 255u) {
    bad = true;
    return;
  }
  const uint32_t m = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
  if (m) atomicAdd(&s_bins[e], (unsigned long long)m);
}

// One weight by both paths (tails).
__device__ __forceinline__ void absmean_one(float w, unsigned long long& lo, uint32_t& hi,
                                            unsigned long long* s_bins, bool& bad) {
  bool out = false;
  const unsigned long long v = absmean_fast(w, 0ull, out);
  lo += v;
  hi += (lo < v) ? 1u : 0u;
  if (out) absmean_slow(w, s_bins, bad);
}

// Ternary threshold T from beta: the least float32 strictly above beta*(0.5+2^-25).
__device__ __forceinline__ float ternary_threshold(float beta) {
  const double tm = __dmul_rn(double(beta), 0.5000000298023223876953125);  // exact
  float T = __double2float_ru(tm);
  if (double(T) == tm) T = __uint_as_float(__float_as_uint(T) + 1u);
  return T;
}

constexpr int kBigWords = 16;  // 512 bits; the sum is below 2^330 units of 2^-149

// Step 3, run by the last CTA: the exact sum rounded once to float64.  All the
// global reads (bins, every CTA's limb slot, the magic word) are issued at once.
// The limbs are in units of 2^(lo_e - 150).  Returns beta in thread 0 (other
// threads: 0).
__device__ float absmean_finalize(AbsAccum* acc, int64_t n, float eps, float* beta_out, int nctas,
                                 unsigned long long* s_binv, unsigned long long* s_limbsum,
                                 unsigned long long* s_wsum, unsigned long long* s_word,
                                 uint32_t* s_big, int* s_flag, uint32_t lo_e = kFastLo) {
  const int t = threadIdx.x;
  for (int i = t; i < kBigWords + 3; i += blockDim.x) s_word[i] = 0ull;
  if (t == 0) *s_flag = 0;
  __syncthreads();
  if (t < 255) {
    const unsigned long long v = __ldcg(&acc->bins[t]);
    s_binv[t] = v;
    if (v) *s_flag = 1;                         // some magnitude outside the fast window
  }
  // sum every CTA's limb slot: warp shuffles, then one value per warp (no
  // contended shared-memory atomics)
  {
    unsigned long long l0 = 0ull, l1 = 0ull, l2 = 0ull;
    for (int c = t; c < nctas; c += blockDim.x) {
      l0 += __ldcg(&acc->slot[c][0]);
      l1 += __ldcg(&acc->slot[c][1]);
      l2 += __ldcg(&acc->slot[c][2]);
    }
    l0 = warp_sum_u64(l0);
    l1 = warp_sum_u64(l1);
    l2 = warp_sum_u64(l2);
    if ((t & 31) == 0) {
      s_wsum[3 * (t >> 5) + 0] = l0;
      s_wsum[3 * (t >> 5) + 1] = l1;
      s_wsum[3 * (t >> 5) + 2] = l2;
    }
  }
  const unsigned int magic = t == 0 ? __ldcg(&acc->magic) : 0u;
  __syncthreads();
  if (t < 3) {
    unsigned long long v = 0ull;
    for (int w = 0; w < int(blockDim.x >> 5); ++w) v += s_wsum[3 * w + t];
    s_limbsum[t] = v;
  }
  __syncthreads();
  const bool fast = *s_flag == 0;
  if (!fast) {
    for (int j = t; j < 258; j += blockDim.x) {
      const unsigned long long w = j < 255 ? s_binv[j] : s_limbsum[j - 255];
      // bins: m * 2^(max(e,1)-150) = m * 2^(max(e,1)-1) units of 2^-149;
      // limb i weighs 2^(32 i) * 2^(lo_e-150) = 2^(32 i + lo_e - 1) units
      const int shift = j < 255 ? (j > 0 ? j : 1) - 1 : 32 * (j - 255) + int(lo_e) - 1;
      if (w) {
        const int wi = shift >> 5, b = shift & 31;
        const unsigned long long lo64 = w << b, hi64 = b ? (w >> (64 - b)) : 0ull;
        atomicAdd(&s_word[wi], lo64 & 0xFFFFFFFFull);
        atomicAdd(&s_word[wi + 1], lo64 >> 32);
        atomicAdd(&s_word[wi + 2], hi64);
      }
    }
  }
  __syncthreads();
  float beta = 0.f;
  if (t == 0) {
    double D = 0.0;
    if (fast) {
      // total = L0 + L1 2^32 + L2 2^64 units of 2^(lo_e-150) (each L < 2^50)
      const unsigned long long L0 = s_limbsum[0], L1 = s_limbsum[1], L2 = s_limbsum[2];
      unsigned long long lo = L0 + (L1 << 32);
      const unsigned long long hi = (L1 >> 32) + L2 + (lo < L0 ? 1ull : 0ull);
      if (hi == 0ull) {
        D = ldexp(__ull2double_rn(lo), int(lo_e) - 150);
      } else {
        const int sh = 64 - __clzll(hi);            // drop sh low bits, keep a sticky bit
        unsigned long long top = (hi << (64 - sh)) | (lo >> sh);
        top |= (lo << (64 - sh)) != 0ull ? 1ull : 0ull;
        D = ldexp(__ull2double_rn(top), sh + int(lo_e) - 150);
      }
    } else {
      unsigned long long carry = 0ull;
      for (int i = 0; i < kBigWords; ++i) {
        const unsigned long long sw = s_word[i] + carry;
        s_big[i] = uint32_t(sw);
        carry = sw >> 32;
      }
      int top = -1;
      for (int i = kBigWords - 1; i >= 0; --i)
        if (s_big[i]) { top = i * 32 + 31 - __clz(s_big[i]); break; }
      if (top >= 0) {
        const int lsb = top - 52 > 0 ? top - 52 : 0;   // lowest bit kept in the mantissa
        const int w0 = lsb >> 5, b0 = lsb & 31;
        unsigned long long mant = ((unsigned long long)s_big[w0] |
                                   (w0 + 1 < kBigWords ? (unsigned long long)s_big[w0 + 1] << 32 : 0ull)) >> b0;
        if (b0 && w0 + 2 < kBigWords) mant |= (unsigned long long)s_big[w0 + 2] << (64 - b0);
        mant &= (1ull << (top - lsb + 1)) - 1ull;      // the bits [lsb, top]
        if (lsb > 0) {                                 // round to nearest, ties to even
          const int rpos = lsb - 1;
          const int rnd = int((s_big[rpos >> 5] >> (rpos & 31)) & 1u);
          bool sticky = (s_big[rpos >> 5] & ((1u << (rpos & 31)) - 1u)) != 0u;
          for (int i = (rpos >> 5) - 1; i >= 0 && !sticky; --i) sticky = s_big[i] != 0u;
          if (rnd && (sticky || (mant & 1ull))) mant += 1ull;  // 2^53 stays exact
        }
        D = ldexp(double(mant), lsb - 149);
      }
    }
    const double d = __ddiv_rn(D, double(n));
    beta = __fadd_rn(__double2float_rn(d), eps);
    *beta_out = beta;
    if (magic != 0u) raise_status(kDevBadWorkspace);
    acc->ticket = 0u;                            // leave the block clear for the next call
    acc->next_chunk = 0u;
  }
  for (int j = t; j < 255; j += blockDim.x)
    if (s_binv[j]) acc->bins[j] = 0ull;
  return beta;
}

__global__ void __launch_bounds__(kAbsThreads, 1)
absmean_kernel(const float* __restrict__ W, int64_t n, float eps, AbsAccum* __restrict__ acc,
               float* __restrict__ beta_out) {
  extern __shared__ __align__(128) unsigned char stage_smem[];
  __shared__ uint64_t full[kAbsStages], empty[kAbsStages];
  __shared__ int s_chunk[kAbsStages];
  __shared__ int s_issued[kAbsStages];   // phases started on full[s] (copies + the stop mark)
  __shared__ unsigned long long s_bins[256];
  __shared__ unsigned long long s_limb[3];
  __shared__ unsigned long long s_word[kBigWords + 3];
  __shared__ uint32_t s_big[kBigWords];
  __shared__ int s_flag;
  __shared__ int s_timeout;
  __shared__ unsigned long long s_binv[255];
  __shared__ unsigned long long s_wsum[3 * (kAbsThreads / 32)];
  __shared__ bool s_last;
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  for (int i = tid; i < 256; i += blockDim.x) s_bins[i] = 0ull;

  unsigned long long lo = 0ull;
  uint32_t hi = 0u;
  bool bad = false;
  const bool tma = aligned(W, 16);
  const int64_t nvec = tma ? (n & ~int64_t(3)) : 0;             // floats read by bulk copies
  const int64_t nch = ceil_div(nvec, kAbsChunkFloats);
  if (tid == 0) {
    s_timeout = 0;
    for (int s = 0; s < kAbsStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kAbsConsumers / 32);
      s_issued[s] = 0;
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kAbsConsumers / 32) {
    // producer warp: lane 0 hands out chunks and issues the copies
    if ((tid & 31) == 0) {
      unsigned int c = atomicAdd(&acc->next_chunk, 1u);
      for (int it = 0;; ++it) {
        const int s = it % kAbsStages;
        if (it >= kAbsStages && !mbar_wait(&empty[s], uint32_t(it / kAbsStages - 1) & 1u)) {
          s_timeout = 1;
          break;
        }
        if (int64_t(c) >= nch) {           // no more work: tell the consumers of stage s
          s_chunk[s] = -1;
          s_issued[s] += 1;
          mbar_arrive(&full[s]);
          break;
        }
        const unsigned int cur = c;
        c = atomicAdd(&acc->next_chunk, 1u);  // the next chunk, while this copy flies
        const int64_t f0 = int64_t(cur) * kAbsChunkFloats;
        const uint32_t bytes = uint32_t(min(int64_t(kAbsChunkFloats), nvec - f0) * 4);
        s_chunk[s] = int(cur);
        s_issued[s] += 1;
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&full[s], bytes);
        bulk_g2s(stage_smem + size_t(s) * kAbsChunkBytes, W + f0, bytes, &full[s]);
      }
    }
  } else {
    // consumer warps
    for (int it = 0;; ++it) {
      const int s = it % kAbsStages;
      if (!mbar_wait(&full[s], uint32_t(it / kAbsStages) & 1u)) {
        s_timeout = 1;
        break;
      }
      const int c = s_chunk[s];
      if (c < 0) break;
      const int cnt4 = int(min(int64_t(kAbsChunkFloats), nvec - int64_t(c) * kAbsChunkFloats) >> 2);
      const float4* src = reinterpret_cast<const float4*>(stage_smem + size_t(s) * kAbsChunkBytes);
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = tid + u * kAbsConsumers;
        v[u] = i < cnt4 ? src[i] : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&empty[s]);   // this warp is done with stage s
      unsigned long long accb = 0ull;
      bool out = false;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        accb = absmean_fast(v[u].x, accb, out);
        accb = absmean_fast(v[u].y, accb, out);
        accb = absmean_fast(v[u].z, accb, out);
        accb = absmean_fast(v[u].w, accb, out);
      }
      lo += accb;
      hi += (lo < accb) ? 1u : 0u;
      if (__any_sync(0xffffffffu, out)) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          absmean_slow(v[u].x, s_bins, bad);
          absmean_slow(v[u].y, s_bins, bad);
          absmean_slow(v[u].z, s_bins, bad);
          absmean_slow(v[u].w, s_bins, bad);
        }
      }
    }
  }
  __syncthreads();
  if (s_timeout) {  // a wait gave up: report, then wait (bounded) for every stage's
    if (tid == 0) {   // last phase so no copy is still writing when the CTA exits
      raise_status(kDevTimeout);
      for (int s = 0; s < kAbsStages; ++s)
        if (s_issued[s] > 0) (void)mbar_wait(&full[s], uint32_t(s_issued[s] - 1) & 1u);
    }
    return;
  }
  // the few weights outside the bulk copies: the unaligned case, or the < 4 past them
  if (blockIdx.x == 0 || !tma)
    for (int64_t j = nvec + tid + (tma ? 0 : int64_t(blockIdx.x) * blockDim.x); j < n;
         j += tma ? blockDim.x : int64_t(gridDim.x) * blockDim.x)
      absmean_one(W[j], lo, hi, s_bins, bad);

  // Exact CTA reduction of the 96-bit accumulators as three 32-bit limbs
  // (each limb sum stays below 2^41).
  const unsigned long long l0 = warp_sum_u64(lo & 0xFFFFFFFFull);
  const unsigned long long l1 = warp_sum_u64(lo >> 32);
  const unsigned long long l2 = warp_sum_u64((unsigned long long)hi);
  if ((tid & 31) == 0) {                  // one slot per warp: no contended atomics
    s_wsum[3 * warp + 0] = l0;
    s_wsum[3 * warp + 1] = l1;
    s_wsum[3 * warp + 2] = l2;
  }
  if (__syncthreads_or(bad) && tid == 0) raise_status(kDevNonFinite);
  for (int i = tid; i < 256; i += blockDim.x)
    if (s_bins[i]) atomicAdd(&acc->bins[i], s_bins[i]);   // rare: weights outside the window
  if (tid < 3) {                          // plain stores into this CTA's own slot
    unsigned long long v = 0ull;
    for (int w = 0; w < kAbsThreads / 32; ++w) v += s_wsum[3 * w + tid];
    acc->slot[blockIdx.x][tid] = v;
  }

  // Last-CTA-done: the CTA whose ticket completes the grid finalizes.
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const unsigned int ticket = atomicAdd(&acc->ticket, 1u);
    if (ticket >= gridDim.x) raise_status(kDevBadWorkspace);
    s_last = (ticket == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  absmean_finalize(acc, n, eps, beta_out, int(gridDim.x), s_binv, s_limb, s_wsum, s_word, s_big,
                   &s_flag);
}

// W [N,K] float32 -> Wq [N,K] int8 codes, grid-stride from thread `tid`.
__device__ __forceinline__ void ternarize_i8_range(const float* __restrict__ W, int64_t n, float T,
                                                   int8_t* __restrict__ Wq, int64_t tid, int64_t nthr) {
  if (aligned(W, 16) && aligned(Wq, 4)) {
    const int64_t n4 = n >> 2;
    for (int64_t i = tid; i < n4; i += nthr) {
      const float4 v = ld_stream_f4(reinterpret_cast<const float4*>(W) + i);
      char4 q;
      q.x = char(trit_code(v.x, T));
      q.y = char(trit_code(v.y, T));
      q.z = char(trit_code(v.z, T));
      q.w = char(trit_code(v.w, T));
      reinterpret_cast<char4*>(Wq)[i] = q;
    }
    for (int64_t j = (n4 << 2) + tid; j < n; j += nthr) Wq[j] = int8_t(trit_code(W[j], T));
  } else {
    for (int64_t j = tid; j < n; j += nthr) Wq[j] = int8_t(trit_code(W[j], T));
  }
}

__global__ void __launch_bounds__(256)
ternarize_i8_kernel(const float* __restrict__ W, int64_t n, const float* __restrict__ beta,
                    int8_t* __restrict__ Wq) {
  ternarize_i8_range(W, n, ternary_threshold(*beta), Wq, int64_t(blockIdx.x) * blockDim.x + threadIdx.x,
                     int64_t(gridDim.x) * blockDim.x);
}

// The packed word g of row `row` (weights 20g .. 20g+19; digit 1 past K).
__device__ __forceinline__ uint32_t ternarize_pack5_word(const float* __restrict__ W, int64_t K,
                                                         float T, bool vec, int64_t row, int64_t g) {
  const int64_t k0 = g * 20;
  const float* wr = W + row * K;
  uint32_t d[20];
  if (vec && k0 + 20 <= K) {
#pragma unroll
    for (int v = 0; v < 5; ++v) {
      const float4 f = ld_stream_f4(reinterpret_cast<const float4*>(wr + k0) + v);
      d[4 * v + 0] = trit_digit(f.x, T);
      d[4 * v + 1] = trit_digit(f.y, T);
      d[4 * v + 2] = trit_digit(f.z, T);
      d[4 * v + 3] = trit_digit(f.w, T);
    }
  } else {
#pragma unroll
    for (int k = 0; k < 20; ++k) d[k] = (k0 + k < K) ? trit_digit(wr[k0 + k], T) : 1u;
  }
  uint32_t word = 0u;
#pragma unroll
  for (int b = 0; b < 4; ++b)
    word |= pack5_digits(d[5 * b], d[5 * b + 1], d[5 * b + 2], d[5 * b + 3], d[5 * b + 4]) << (8 * b);
  return word;
}

// W [N,K] float32 -> Wp [N,ldp] packed bytes, grid-stride from thread `first`
// with stride `nthr`.  One thread per 4 output bytes (20 weights): a 32-bit
// store, and five 128-bit loads when the group is whole.
__device__ __forceinline__ void ternarize_pack5_range(const float* __restrict__ W, int64_t N,
                                                      int64_t K, float T, uint8_t* __restrict__ Wp,
                                                      int64_t ldp, int64_t first, int64_t nthr) {
  const int64_t words = ldp >> 2;
  const int64_t total = N * words;
  const bool small = total < (int64_t(1) << 32);
  const bool vec = aligned(W, 16) && (K & 3) == 0;
  for (int64_t i = first; i < total; i += nthr) {
    int64_t row, g;
    split_index(i, words, small, row, g);
    *reinterpret_cast<uint32_t*>(Wp + row * ldp + 4 * g) = ternarize_pack5_word(W, K, T, vec, row, g);
  }
}

__global__ void __launch_bounds__(256)
ternarize_pack5_kernel(const float* __restrict__ W, int64_t N, int64_t K,
                       const float* __restrict__ beta, uint8_t* __restrict__ Wp, int64_t ldp) {
  ternarize_pack5_range(W, N, K, ternary_threshold(*beta), Wp, ldp,
                        int64_t(blockIdx.x) * blockDim.x + threadIdx.x, int64_t(gridDim.x) * blockDim.x);
}

}  // namespace bl
