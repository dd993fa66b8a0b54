// RMSNorm fused into the per-row activation quantization of the next BitLinear.
//
// "ultragraph -- when the graph is the 1-bit LLM, part 2", section "attention,
// as graph ops": RMSNorm(x) = x / sqrt((1/d) sum_i x_i^2 + eps) * g; the pre-norm
// block of "ultragraph-1bit 0.12.0" (PyPI), "x = x + mha(norm1(x))", feeds the
// normalized rows to the BitLinear layers, whose first step is the per-row
// absmax quantization of section "the bytes".  One CTA per row, one read of x:
//
//   1. the row goes to shared memory; the largest exponent of |x| is found;
//   2. the mean of squares is exact: every square m^2 2^(2E-300) of a float32
//      (m its 24-bit significand, E its exponent, at least 1) is an integer in
//      units of 2^-298.  Each thread adds its squares into a 192-bit fixed-point
//      window whose units are 2^(2 Emax - 426): a square with 2 (Emax - E) <= 126
//      lands there exactly (at most 48 + 126 + 17 bits, so no overflow for
//      K <= 2^17); the rare smaller ones (|x| below 2^-63 |x|max) go to
//      per-exponent bins in shared memory.  The CTA adds the windows (192-bit
//      sums with carries), places window and bins in a 640-bit integer and rounds
//      it once to float64 (nearest, ties to even); then ms = float32(S / d) with
//      the division in float64, as the definition reads;
//   3. r = sqrt(ms + eps_norm) and y = (x / r) * g in float32 (IEEE, no FMA);
//   4. s = max|y| / 127 + eps and x_q = clip(round(y / s), -127, 127), exactly as
//      bl_quantize_act.
#pragma once

#include "act_quant.cuh"
#include "common.cuh"

namespace bl {

constexpr int kRnThreads = 256;
constexpr int kRnBigWords = 20;               // 640 bits: squares reach 2^573 units of 2^-298
constexpr int64_t kRnMaxK = 49152;            // row in shared memory (192 KB)

__device__ __forceinline__ void add192(unsigned long long& a0, unsigned long long& a1, unsigned long long& a2,
                                       unsigned long long b0, unsigned long long b1, unsigned long long b2) {
  asm("add.cc.u64 %0, %0, %3;\n\taddc.cc.u64 %1, %1, %4;\n\taddc.u64 %2, %2, %5;"
      : "+l"(a0), "+l"(a1), "+l"(a2)
      : "l"(b0), "l"(b1), "l"(b2));
}

// Adds the 64-bit value v << shift (shift >= 0) into the little-endian 32-bit
// word array `w` (64-bit accumulators per 32-bit word; carries resolved later).
__device__ __forceinline__ void big_add(unsigned long long* w, unsigned long long v, int shift) {
  if (!v) return;
  const int wi = shift >> 5, b = shift & 31;
  const unsigned long long lo = v << b, hi = b ? (v >> (64 - b)) : 0ull;
  w[wi] += lo & 0xFFFFFFFFull;
  w[wi + 1] += lo >> 32;
  w[wi + 2] += hi;
}

__global__ void __launch_bounds__(kRnThreads)
rmsnorm_quant_kernel(const float* __restrict__ X, int64_t K, const float* __restrict__ g, float eps_norm,
                     float eps, int8_t* __restrict__ Xq, int64_t ldq, float* __restrict__ s_out) {
  extern __shared__ __align__(16) float xs[];
  __shared__ unsigned long long s_bins[2][256];
  __shared__ unsigned long long s_win[kRnThreads / 32][3];
  __shared__ uint32_t s_emax[kRnThreads / 32];
  __shared__ float s_red[kRnThreads / 32];
  __shared__ int s_slow;
  __shared__ float s_r, s_scale;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t m = blockIdx.x;
  const float* xr = X + m * K;
  int8_t* qr = Xq + m * ldq;

  // 1. row into shared memory, largest biased exponent, finiteness
  if (tid == 0) s_slow = 0;
  for (int i = tid; i < 512; i += kRnThreads) (&s_bins[0][0])[i] = 0ull;
  uint32_t emax = 0;
  bool bad = false;
  const bool vec = aligned(xr, 16) && (K & 3) == 0;
  if (vec) {
    for (int64_t i = tid; i < (K >> 2); i += kRnThreads) {
      const float4 v = ld_stream_f4(reinterpret_cast<const float4*>(xr) + i);
      reinterpret_cast<float4*>(xs)[i] = v;
      const uint32_t e = max(max(__float_as_uint(v.x) & 0x7FFFFFFFu, __float_as_uint(v.y) & 0x7FFFFFFFu),
                             max(__float_as_uint(v.z) & 0x7FFFFFFFu, __float_as_uint(v.w) & 0x7FFFFFFFu));
      emax = max(emax, e);
    }
  } else {
    for (int64_t i = tid; i < K; i += kRnThreads) {
      const float v = xr[i];
      xs[i] = v;
      emax = max(emax, __float_as_uint(v) & 0x7FFFFFFFu);
    }
  }
  bad = (emax >> 23) == 255u;                   // Inf or NaN: the largest magnitude bits say so
  for (int o = 16; o > 0; o >>= 1) emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  if (lane == 0) s_emax[warp] = emax;
  if (__syncthreads_or(bad)) {
    if (tid == 0) raise_status(kDevNonFinite);
  }
  for (int w = 0; w < kRnThreads / 32; ++w) emax = max(emax, s_emax[w]);
  const int Emax = max(int(emax >> 23), 1);

  // 2. exact sum of squares: 192-bit window, units 2^(2 Emax - 426)
  unsigned long long a0 = 0ull, a1 = 0ull, a2 = 0ull;
  for (int64_t i = tid; i < K; i += kRnThreads) {
    const uint32_t u = __float_as_uint(xs[i]) & 0x7FFFFFFFu;
    const uint32_t e = u >> 23;
    const unsigned long long mm = (u & 0x7FFFFFu) | (e ? 0x800000u : 0u);
    if (!mm) continue;
    const int E = max(int(e), 1);
    const unsigned long long sq = mm * mm;      // < 2^48
    const int sh = 2 * (Emax - E);
    if (sh > 126) {                              // far below the largest |x|: exact bins
      atomicAdd(&s_bins[0][E], sq & 0xFFFFFFull);
      atomicAdd(&s_bins[1][E], sq >> 24);
      s_slow = 1;
      continue;
    }
    const int sft = 126 - sh;                    // the square's lowest bit in the window
    unsigned long long p0 = 0ull, p1 = 0ull, p2 = 0ull;
    if (sft < 64) {
      p0 = sq << sft;
      p1 = sft ? (sq >> (64 - sft)) : 0ull;
    } else {
      const int s2 = sft - 64;
      p1 = sq << s2;
      p2 = s2 ? (sq >> (64 - s2)) : 0ull;
    }
    add192(a0, a1, a2, p0, p1, p2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long b0 = __shfl_xor_sync(0xffffffffu, a0, o);
    const unsigned long long b1 = __shfl_xor_sync(0xffffffffu, a1, o);
    const unsigned long long b2 = __shfl_xor_sync(0xffffffffu, a2, o);
    add192(a0, a1, a2, b0, b1, b2);
  }
  if (lane == 0) {
    s_win[warp][0] = a0;
    s_win[warp][1] = a1;
    s_win[warp][2] = a2;
  }
  __syncthreads();
  if (tid == 0) {
    unsigned long long w0 = 0ull, w1 = 0ull, w2 = 0ull;
    for (int w = 0; w < kRnThreads / 32; ++w) add192(w0, w1, w2, s_win[w][0], s_win[w][1], s_win[w][2]);
    // the exact sum as a 640-bit integer in units of 2^-298
    unsigned long long acc[kRnBigWords + 3];
    for (int i = 0; i < kRnBigWords + 3; ++i) acc[i] = 0ull;
    const int off = 2 * Emax - 128;              // window unit 2^(2 Emax - 426) = 2^off units
    if (off >= 0) {
      big_add(acc, w0, off);
      big_add(acc, w1, off + 64);
      big_add(acc, w2, off + 128);
    } else {                                     // the low -off bits of the window are zero
      const int r = -off;                        // 0 < r <= 126
      unsigned long long v0, v1, v2;
      if (r < 64) {
        v0 = (w0 >> r) | (w1 << (64 - r));
        v1 = (w1 >> r) | (w2 << (64 - r));
        v2 = w2 >> r;
      } else {
        const int r2 = r - 64;
        v0 = r2 ? ((w1 >> r2) | (w2 << (64 - r2))) : w1;
        v1 = r2 ? (w2 >> r2) : w2;
        v2 = 0ull;
      }
      big_add(acc, v0, 0);
      big_add(acc, v1, 64);
      big_add(acc, v2, 128);
    }
    if (s_slow)
      for (int E = 1; E < 256; ++E) {
        big_add(acc, s_bins[0][E], 2 * E - 2);
        big_add(acc, s_bins[1][E], 2 * E - 2 + 24);
      }
    uint32_t big[kRnBigWords];
    unsigned long long carry = 0ull;
    for (int i = 0; i < kRnBigWords; ++i) {
      const unsigned long long v = acc[i] + carry;
      big[i] = uint32_t(v);
      carry = v >> 32;
    }
    double D = 0.0;
    int top = -1;
    for (int i = kRnBigWords - 1; i >= 0; --i)
      if (big[i]) {
        top = i * 32 + 31 - __clz(big[i]);
        break;
      }
    if (top >= 0) {
      const int lsb = top - 52 > 0 ? top - 52 : 0;
      const int q0 = lsb >> 5, b0 = lsb & 31;
      unsigned long long mant = ((unsigned long long)big[q0] |
                                 (q0 + 1 < kRnBigWords ? (unsigned long long)big[q0 + 1] << 32 : 0ull)) >> b0;
      if (b0 && q0 + 2 < kRnBigWords) mant |= (unsigned long long)big[q0 + 2] << (64 - b0);
      mant &= (1ull << (top - lsb + 1)) - 1ull;
      if (lsb > 0) {                             // round to nearest, ties to even
        const int rp = lsb - 1;
        const int rnd = int((big[rp >> 5] >> (rp & 31)) & 1u);
        bool sticky = (big[rp >> 5] & ((1u << (rp & 31)) - 1u)) != 0u;
        for (int i = (rp >> 5) - 1; i >= 0 && !sticky; --i) sticky = big[i] != 0u;
        if (rnd && (sticky || (mant & 1ull))) mant += 1ull;
      }
      D = ldexp(double(mant), lsb - 298);
    }
    const float ms = __double2float_rn(__ddiv_rn(D, double(K)));
    s_r = __fsqrt_rn(__fadd_rn(ms, eps_norm));
  }
  __syncthreads();

  // 3. y = (x / r) * g, kept in shared memory; 4. the row's absmax
  const float r = s_r;
  float amax = 0.f;
  for (int64_t i = tid; i < K; i += kRnThreads) {
    const float y = __fmul_rn(__fdiv_rn(xs[i], r), g[i]);
    xs[i] = y;
    amax = fmaxf(amax, fabsf(y));
  }
  amax = warp_max(amax);
  if (lane == 0) s_red[warp] = amax;
  __syncthreads();
  if (tid < 32) {
    float v = tid < kRnThreads / 32 ? s_red[tid] : 0.f;
    v = warp_max(v);
    if (tid == 0) {
      const float s = __fadd_rn(__fdiv_rn(v, float(kActQmax)), eps);
      s_scale = s;
      s_out[m] = s;
    }
  }
  __syncthreads();
  const float s = s_scale;
  const float rc = act_recip(s);
  for (int64_t i = tid; i < K; i += kRnThreads) qr[i] = act_code_fast(xs[i], s, rc);
  for (int64_t i = K + tid; i < ldq; i += kRnThreads) qr[i] = 0;
}

}  // namespace bl
