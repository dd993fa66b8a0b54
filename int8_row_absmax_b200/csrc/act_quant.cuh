// Per-row (per-token) absmax int8 quantization of activations.
//
// "ultragraph -- when the graph is the 1-bit LLM, part 2", section "the bytes",
// and the per-token fix in section "attention, as graph ops":
//   s = max_i |x_i| / 127 + eps,   x_q = clip(round(x / s), -127, 127).
// One scale per row, so no row's codes depend on another row.  All float32,
// IEEE division, round half to even (rintf), in the written order.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "trit_table.cuh"

namespace bl {

constexpr int kActThreads = 256;

__device__ __forceinline__ int8_t act_code(float x, float s) {
  float q = rintf(__fdiv_rn(x, s));
  q = fminf(fmaxf(q, -float(kActQmax)), float(kActQmax));
  return int8_t(int(q));
}

// act_code kept out of line: the rare near-tie path of act_code_fast.
__device__ __noinline__ int act_code_slow(float x, float s) { return act_code(x, s); }

// Reciprocal of the row scale for act_code_fast, or 0 when the fast path is not
// safe for this scale (s not a normal float, or 1/s not a normal float).
__device__ __forceinline__ float act_recip(float s) {
  const float r = __frcp_rn(s);
  return (s >= 1.17549435e-38f && r >= 1.17549435e-38f && r <= 1.0e37f) ? r : 0.f;
}

// The same code as act_code, with one multiply instead of the IEEE division in
// all but near-tie cases.  For |x| <= 127 s, y' = x * RN(1/s) differs from the
// real quotient y = x / s by at most 1.5 ulp(y) <= 1.5 * 2^-17 < 2^-16, and
// float32(y) is within 2^-18 of y.  So unless y' lies within 2^-15 of a
// half-integer, y, float32(y) and y' all round to the same integer; the rare
// near-tie values take the exact division.  The rounding itself is t = y +
// 1.5 * 2^23 (round to nearest even, exact for |y| <= 127), so the code is the
// low byte of t's bits (two's complement) and no conversion instruction is
// needed.  Returned in the low byte.
__device__ __forceinline__ uint32_t act_code_bits(float x, float s, float r) {
  const float y = fminf(fmaxf(__fmul_rn(x, r), -float(kActQmax)), float(kActQmax));
  const float t = __fadd_rn(y, 12582912.0f);
  const float d = __fsub_rn(y, __fsub_rn(t, 12582912.0f));
  if (r == 0.f || fabsf(fabsf(d) - 0.5f) < 3.0517578125e-05f)
    return uint32_t(uint8_t(int8_t(act_code_slow(x, s))));
  return __float_as_uint(t) & 0xFFu;
}
__device__ __forceinline__ int8_t act_code_fast(float x, float s, float r) {
  return int8_t(uint8_t(act_code_bits(x, s, r)));
}
// act_code_bits without its branch: the caller redoes the codes with act_code
// when `tie` comes back set (near a half-integer, or r == 0).
__device__ __forceinline__ uint32_t act_code_try(float x, float r, bool& tie) {
  const float y = fminf(fmaxf(__fmul_rn(x, r), -float(kActQmax)), float(kActQmax));
  const float t = __fadd_rn(y, 12582912.0f);
  const float d = __fsub_rn(y, __fsub_rn(t, 12582912.0f));
  tie |= fabsf(fabsf(d) - 0.5f) < 3.0517578125e-05f;
  return __float_as_uint(t) & 0xFFu;
}
// Whether act_code_try's code for x may differ from act_code: the product
// within 2^-15 of a half-integer, or no usable reciprocal (r == 0).  A group
// whose `tie` came back set redoes only these elements with the exact division.
__device__ __forceinline__ bool act_near_tie(float x, float r) {
  if (r == 0.f) return true;
  const float y = fminf(fmaxf(__fmul_rn(x, r), -float(kActQmax)), float(kActQmax));
  const float t = __fadd_rn(y, 12582912.0f);
  const float d = __fsub_rn(y, __fsub_rn(t, 12582912.0f));
  return fabsf(fabsf(d) - 0.5f) < 3.0517578125e-05f;
}
// The exact code of x for a product x * r within 2^-15 of a half-integer
// (r = act_recip(s) != 0), with no division.  Let a = |x|, n = floor(RN(a r))
// and h = n + 1/2; the exact quotient a / s lies within 2^-15 + 1.5 ulp of h,
// so RN(a / s) is h, a float below h (code n) or a float above h (code n + 1).
// For h <= 127.5 the last significand bit of h is 0, so the two midpoints
// h -+ ulp(h)/2 round to h: RN(a / s) = h exactly when s (h - u/2) <= a <=
// s (h + u/2), u = ulp(h).  Those bounds are products of a 24-bit and a 25-bit
// significand, exact in float64, so two comparisons decide; RN(a / s) = h then
// rounds half to even.  (For h = 1/2 the float below h is only ulp(h)/2 away,
// but every quotient at or below h then has code 0 either way.)  The code of
// -x is minus that of x.
__device__ __forceinline__ uint32_t act_code_tie_exact(float x, float s, float r) {
  const float a = fabsf(x);
  const float yq = fminf(__fmul_rn(a, r), float(kActQmax));
  const float n = floorf(yq);
  const float h = __fadd_rn(n, 0.5f);
  const int eh = (int((__float_as_uint(h) >> 23) & 0xFFu)) - 127;   // h >= 0.5: normal
  const double hu = __longlong_as_double(int64_t(1023 + eh - 24) << 52);   // ulp(h) / 2 = 2^(eh-24)
  const double ds = double(s), da = double(a);
  const double lo = ds * (double(h) - hu), hi = ds * (double(h) + hu);
  const int ni = int(n);
  int q = da < lo ? ni : (da > hi ? ni + 1 : ni + (ni & 1));
  q = q > kActQmax ? kActQmax : q;
  return uint32_t(uint8_t(int8_t(x < 0.f ? -q : q)));
}

// Codes of N activations x[0..N-1] of a row whose scale s came from that row's
// own max|x| (so |x| <= max|x| <= 127 s, and the product x RN(1/s) stays below
// 127.5: no clamp is needed before rounding); elements from `valid` on are not
// part of the row (code 0; the caller passes them as 0).  Each code is returned
// in the LOW BYTE of c[e] (the upper bytes are not cleared: pack with
// byte_perm).  Per element: one multiply, the round-to-nearest-even of
// act_code_try and the distance of the product from the nearest half-integer,
// of which the unit keeps only the minimum.  A unit whose minimum lies within
// 2^-15 finds its near-tie elements: one takes the division-free exact code of
// act_code_tie_exact (inline: per-CTA quantizations of the same row take the
// same branches in every CTA, and an out-of-line routine costs its instruction
// fetches each time); two or more, or no usable reciprocal (rc == 0), take the
// exact division per element.
template <int N>
__device__ __forceinline__ void act_codes_n(const float* x, int valid, float s, float rc, uint32_t* c) {
  float dmin = 1.0f;
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const float y = __fmul_rn(x[e], rc);
    const float t = __fadd_rn(y, 12582912.0f);
    const float d = __fsub_rn(y, __fsub_rn(t, 12582912.0f));
    dmin = fminf(dmin, fabsf(__fsub_rn(fabsf(d), 0.5f)));
    c[e] = __float_as_uint(t);
  }
  if (rc == 0.f || dmin < 3.0517578125e-05f) {
    uint32_t near = 0u;
#pragma unroll
    for (int e = 0; e < N; ++e)
      if (e < valid && act_near_tie(x[e], rc)) near |= 1u << e;
    if (rc == 0.f || (near & (near - 1u)) != 0u) {
#pragma unroll
      for (int e = 0; e < N; ++e)
        if (e < valid && (rc == 0.f || ((near >> e) & 1u)))
          c[e] = uint32_t(uint8_t(int8_t(act_code_slow(x[e], s))));
    } else if (near) {
      const int te = __ffs(int(near)) - 1;
      float xt = x[0];
#pragma unroll
      for (int e = 1; e < N; ++e)
        if (e == te) xt = x[e];
      const uint32_t ce = act_code_tie_exact(xt, s, rc);
#pragma unroll
      for (int e = 0; e < N; ++e)
        if (e == te) c[e] = ce;
    }
  }
  if (valid < N) {
#pragma unroll
    for (int e = 0; e < N; ++e)
      if (e >= valid) c[e] = 0u;
  }
}

// The low bytes of four code words, little-endian, in one word.
__device__ __forceinline__ uint32_t pack_code_bytes(uint32_t c0, uint32_t c1, uint32_t c2, uint32_t c3) {
  return __byte_perm(__byte_perm(c0, c1, 0x0040), __byte_perm(c2, c3, 0x0040), 0x5410);
}

// Four codes packed little-endian into one word.
__device__ __forceinline__ uint32_t act_codes4(float4 v, float s, float r) {
  return __byte_perm(__byte_perm(act_code_bits(v.x, s, r), act_code_bits(v.y, s, r), 0x0040),
                     __byte_perm(act_code_bits(v.z, s, r), act_code_bits(v.w, s, r), 0x0040), 0x5410);
}

// One CTA per row: pass 1 finds max|x| (warp shuffles, then across warps), pass
// 2 re-reads the row (an L1/L2 hit) and writes the codes.  Row stride of X is K;
// Xq has stride ldq >= K and its bytes [K, ldq) are written as 0.
__global__ void __launch_bounds__(kActThreads)
act_quant_kernel(const float* __restrict__ X, int64_t K, float eps, int8_t* __restrict__ Xq,
                 int64_t ldq, float* __restrict__ s_out) {
  __shared__ float s_red[kActThreads / 32];
  __shared__ float s_scale;
  const int64_t m = blockIdx.x;
  const float* xr = X + m * K;
  int8_t* qr = Xq + m * ldq;
  const bool vec = aligned(xr, 16) && aligned(qr, 4);
  const int64_t K4 = vec ? (K >> 2) : 0;

  float amax = 0.f;
  bool bad = false;
  for (int64_t i = threadIdx.x; i < K4; i += kActThreads) {
    const float4 v = reinterpret_cast<const float4*>(xr)[i];
    const float a = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
    bad |= !(fabsf(v.x) <= 3.402823466e38f) | !(fabsf(v.y) <= 3.402823466e38f) |
           !(fabsf(v.z) <= 3.402823466e38f) | !(fabsf(v.w) <= 3.402823466e38f);
    amax = fmaxf(amax, a);
  }
  for (int64_t i = (K4 << 2) + threadIdx.x; i < K; i += kActThreads) {
    const float a = fabsf(xr[i]);
    bad |= !(a <= 3.402823466e38f);
    amax = fmaxf(amax, a);
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
  if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(kDevNonFinite);
  if (threadIdx.x < 32) {
    float v = threadIdx.x < kActThreads / 32 ? s_red[threadIdx.x] : 0.f;
    v = warp_max(v);
    if (threadIdx.x == 0) {
      const float s = __fadd_rn(__fdiv_rn(v, float(kActQmax)), eps);
      s_scale = s;
      s_out[m] = s;
    }
  }
  __syncthreads();
  const float s = s_scale;
  const float r = act_recip(s);

  for (int64_t i = threadIdx.x; i < K4; i += kActThreads) {
    const float4 v = reinterpret_cast<const float4*>(xr)[i];
    reinterpret_cast<uint32_t*>(qr)[i] = act_codes4(v, s, r);
  }
  for (int64_t i = (K4 << 2) + threadIdx.x; i < K; i += kActThreads) qr[i] = act_code_fast(xr[i], s, r);
  for (int64_t i = K + threadIdx.x; i < ldq; i += kActThreads) qr[i] = 0;
}

// Single-pass variant for rows that fit in registers: each thread keeps its
// VPT float4 of the row between the max and the quantization, so X is read
// from memory exactly once.  Needs X rows 16-byte aligned (K % 4 == 0) and Xq
// rows 4-byte aligned; K <= VPT * 4 * kActThreads.
template <int VPT>
__global__ void __launch_bounds__(kActThreads)
act_quant_reg_kernel(const float* __restrict__ X, int64_t K, float eps, int8_t* __restrict__ Xq,
                     int64_t ldq, float* __restrict__ s_out) {
  __shared__ float s_red[kActThreads / 32];
  __shared__ float s_scale;
  const int64_t m = blockIdx.x;
  const float4* xr = reinterpret_cast<const float4*>(X + m * K);
  int8_t* qr = Xq + m * ldq;
  const int K4 = int(K >> 2);
  float4 v[VPT];
  float amax = 0.f;
  bool bad = false;
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int i = threadIdx.x + u * kActThreads;
    v[u] = i < K4 ? ld_stream_f4(xr + i) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float a = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
    bad |= !(a <= 3.402823466e38f) | (v[u].x != v[u].x) | (v[u].y != v[u].y) | (v[u].z != v[u].z) |
           (v[u].w != v[u].w);
    amax = fmaxf(amax, a);
  }
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = amax;
  if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(kDevNonFinite);
  if (threadIdx.x < 32) {
    float w = threadIdx.x < kActThreads / 32 ? s_red[threadIdx.x] : 0.f;
    w = warp_max(w);
    if (threadIdx.x == 0) {
      const float s = __fadd_rn(__fdiv_rn(w, float(kActQmax)), eps);
      s_scale = s;
      s_out[m] = s;
    }
  }
  __syncthreads();
  const float s = s_scale;
  const float r = act_recip(s);
#pragma unroll
  for (int u = 0; u < VPT; ++u) {
    const int i = threadIdx.x + u * kActThreads;
    if (i < K4) reinterpret_cast<uint32_t*>(qr)[i] = act_codes4(v[u], s, r);
  }
  for (int64_t i = K + threadIdx.x; i < ldq; i += kActThreads) qr[i] = 0;
}

// The same codes, written in the decode order of trit_table.cuh (positions
// dorder_pos(k); bytes [K, ldq) of the order's row are 0), for the swapped
// tensor-core GEMM.  One CTA of 512 threads per row.  With G > 0 the row fits
// in registers (at most G packed words of 20 activations per thread): each
// thread issues all its loads at once, takes the max, and after the CTA's
// reduction turns the same registers into its words' five code words each, so
// X is read once.  G = 0: two passes over the row (max, then codes).  It lets
// the next kernel on the stream begin its prologue at once (programmatic
// dependent launch).
constexpr int kActDoThreads = 512;

// Codes of one packed word's 20 activations (c[e] = code of x[e]) as the five
// decode-order words at dst.
__device__ __forceinline__ void store_dorder_word(uint32_t* dst, const uint32_t* c) {
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = pack_code_bytes(c[5 * i], c[5 * i + 1], c[5 * i + 2], c[5 * i + 3]);
  dst[4] = pack_code_bytes(c[4], c[9], c[14], c[19]);
}

template <int G>
__global__ void __launch_bounds__(kActDoThreads)
act_quant_dorder_kernel(const float* __restrict__ X, int64_t K, float eps, int8_t* __restrict__ Xq,
                        int64_t ldq, float* __restrict__ s_out) {
  __shared__ float s_red[kActDoThreads / 32];
  __shared__ float s_scale;
  griddep_wait();
  griddep_launch_dependents();
  const int tid = threadIdx.x;
  const int64_t m = blockIdx.x;
  const float* xr = X + m * K;
  uint32_t* qw = reinterpret_cast<uint32_t*>(Xq + m * ldq);
  const bool vec = aligned(xr, 16) && (K & 3) == 0;
  const int64_t ngrp = (K + 19) / 20;
  float amax = 0.f;
  bool bad = false;
  float v[G > 0 ? G : 1][20];
  if constexpr (G > 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int64_t k0 = 20 * (int64_t(tid) + int64_t(g) * kActDoThreads);
      if (vec && k0 + 20 <= K) {
#pragma unroll
        for (int q = 0; q < 5; ++q) {
          const float4 f = reinterpret_cast<const float4*>(xr + k0)[q];
          v[g][4 * q] = f.x;
          v[g][4 * q + 1] = f.y;
          v[g][4 * q + 2] = f.z;
          v[g][4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 20; ++e) v[g][e] = k0 + e < K ? xr[k0 + e] : 0.f;
      }
    }
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int e = 0; e < 20; ++e) {
        const float a = fabsf(v[g][e]);
        bad |= !(a <= 3.402823466e38f);
        amax = fmaxf(amax, a);
      }
  } else {
    const int64_t K4 = vec ? (K >> 2) : 0;
    for (int64_t i = tid; i < K4; i += kActDoThreads) {
      const float4 f = reinterpret_cast<const float4*>(xr)[i];
      const float a = fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w)));
      bad |= !(a <= 3.402823466e38f) | (f.x != f.x) | (f.y != f.y) | (f.z != f.z) | (f.w != f.w);
      amax = fmaxf(amax, a);
    }
    for (int64_t i = (K4 << 2) + tid; i < K; i += kActDoThreads) {
      const float a = fabsf(xr[i]);
      bad |= !(a <= 3.402823466e38f);
      amax = fmaxf(amax, a);
    }
  }
  amax = warp_max(amax);
  if ((tid & 31) == 0) s_red[tid >> 5] = amax;
  if (__syncthreads_or(bad) && tid == 0) raise_status(kDevNonFinite);
  if (tid < 32) {
    float w = tid < kActDoThreads / 32 ? s_red[tid] : 0.f;
    w = warp_max(w);
    if (tid == 0) {
      const float sc = __fadd_rn(__fdiv_rn(w, float(kActQmax)), eps);
      s_scale = sc;
      s_out[m] = sc;
    }
  }
  __syncthreads();
  const float s = s_scale;
  const float rc = act_recip(s);
  if constexpr (G > 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const int64_t gi = int64_t(tid) + int64_t(g) * kActDoThreads;
      if (gi >= ngrp) break;
      const int64_t k0 = 20 * gi;
      uint32_t c[20];
      act_codes_n<20>(v[g], int(min(int64_t(20), K - k0)), s, rc, c);
      store_dorder_word(qw + 5 * gi, c);
    }
  } else {
    for (int64_t gi = tid; gi < ngrp; gi += kActDoThreads) {
      const int64_t k0 = 20 * gi;
      float xv[20];
      if (vec && k0 + 20 <= K) {
#pragma unroll
        for (int q = 0; q < 5; ++q) {
          const float4 f = reinterpret_cast<const float4*>(xr + k0)[q];
          xv[4 * q] = f.x;
          xv[4 * q + 1] = f.y;
          xv[4 * q + 2] = f.z;
          xv[4 * q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 20; ++e) xv[e] = k0 + e < K ? xr[k0 + e] : 0.f;
      }
      uint32_t c[20];
      act_codes_n<20>(xv, int(min(int64_t(20), K - k0)), s, rc, c);
      store_dorder_word(qw + 5 * gi, c);
    }
  }
  for (int64_t i = 5 * ngrp + tid; i < (ldq >> 2); i += kActDoThreads) qw[i] = 0u;
}

// The decode-order quantizer for M rows of K (the register form when the row fits).
inline void launch_act_quant_dorder(const float* X, int64_t M, int64_t K, float eps, int8_t* Xq, int64_t ldq,
                                    float* s, cudaStream_t st) {
  const int64_t ngrp = (K + 19) / 20;
  const unsigned g = unsigned(M);
  if (ngrp <= kActDoThreads) act_quant_dorder_kernel<1><<<g, kActDoThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else if (ngrp <= 2 * kActDoThreads) act_quant_dorder_kernel<2><<<g, kActDoThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
  else act_quant_dorder_kernel<0><<<g, kActDoThreads, 0, st>>>(X, K, eps, Xq, ldq, s);
}

// Given codes [M, ldx] in natural order -> the decode order [M, ldd] (ldd % 4
// == 0, ldd >= dorder_len(K)); one thread per output word.
__global__ void xq_dorder_kernel(const int8_t* __restrict__ Xq, int64_t ldx, int64_t M, int64_t K,
                                 int8_t* __restrict__ Xd, int64_t ldd) {
  griddep_wait();
  griddep_launch_dependents();
  const int64_t wpr = ldd >> 2;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < M * wpr;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t m = i / wpr, wi = i - m * wpr;
    const int64_t g = wi / 5, q = wi - 5 * g;
    const int8_t* xr = Xq + m * ldx;
    uint32_t v = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t k = q < 4 ? 5 * (4 * g + q) + e : 5 * (4 * g + e) + 4;
      if (k < K) v |= uint32_t(uint8_t(xr[k])) << (8 * e);
    }
    reinterpret_cast<uint32_t*>(Xd + m * ldd)[wi] = v;
  }
}

}  // namespace bl
