// Shared device helpers for the BitLinear kernels (one translation unit).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "bitlinear.h"

namespace bl {

// Per-device status word.  Kernels OR flags in; bl_sync_status reads and clears.
enum : unsigned int { kDevTimeout = 1u, kDevNonFinite = 2u, kDevBadWorkspace = 4u };
__device__ unsigned int g_status = 0u;

__device__ __forceinline__ void raise_status(unsigned int f) { atomicOr(&g_status, f); }

constexpr int kActQmax = 127;          // symmetric int8 range [-127, 127]
constexpr int64_t kMaxK = 131072;      // 127 * K < 2^24: every accumulator exact in float32

__host__ __device__ constexpr int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ constexpr int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

__device__ __forceinline__ bool aligned(const void* p, uintptr_t a) {
  return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0;
}

// Streaming 128-bit load that does not allocate in L1 (data is read once).
__device__ __forceinline__ float4 ld_stream_f4(const float4* p) {
  float4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// (row, column) of flat item i in rows of `per_row` items; 32-bit division
// when the item count allows (64-bit integer division is a long software
// routine on the GPU).
__device__ __forceinline__ void split_index(int64_t i, int64_t per_row, bool small, int64_t& row,
                                            int64_t& col) {
  if (small) {
    const uint32_t r = uint32_t(i) / uint32_t(per_row);
    row = r;
    col = int64_t(uint32_t(i) - r * uint32_t(per_row));
  } else {
    row = i / per_row;
    col = i - row * per_row;
  }
}

// Ternary digit d = t + 1 in {0,1,2} of a weight against the precomputed
// threshold T (see weight_quant.cuh): |w| >= T means round(w / beta) != 0.
__device__ __forceinline__ uint32_t trit_digit(float w, float T) {
  return fabsf(w) >= T ? (w > 0.f ? 2u : 0u) : 1u;
}
__device__ __forceinline__ int trit_code(float w, float T) {
  return fabsf(w) >= T ? (w > 0.f ? 1 : -1) : 0;
}

// Byte of five digits, little-endian base 3: d0 + 3 d1 + 9 d2 + 27 d3 + 81 d4.
__device__ __forceinline__ uint32_t pack5_digits(uint32_t d0, uint32_t d1, uint32_t d2,
                                                 uint32_t d3, uint32_t d4) {
  return d0 + 3u * (d1 + 3u * (d2 + 3u * (d3 + 3u * d4)));
}

// The five trits of a packed byte: t_k = floor(b / 3^k) mod 3 - 1.
__device__ __forceinline__ void unpack5_byte(uint32_t b, int t[5]) {
#pragma unroll
  for (int k = 0; k < 5; ++k) {
    t[k] = int(b % 3u) - 1;
    b /= 3u;
  }
}

}  // namespace bl
