// Dense trit packing: five trits per byte, byte = sum_{k<5} (t_k + 1) * 3^k.
//
// "ultragraph-1bit 0.12.0" (PyPI), sections "A whole ternary GPT" and "Layout"
// (5 ternary values per byte, ~1.6 bits/weight).  Trits run along K in order;
// trits past K are 0, so a whole padding byte is 121; rows are ldp bytes apart.
#pragma once

#include "common.cuh"

namespace bl {

// Wq [N,K] int8 (contiguous) -> Wp [N,ldp].  One thread per 4 output bytes.
__global__ void __launch_bounds__(256)
pack5_kernel(const int8_t* __restrict__ Wq, int64_t N, int64_t K, uint8_t* __restrict__ Wp,
             int64_t ldp) {
  const int64_t words = ldp >> 2;
  const int64_t total = N * words;
  const bool small = total < (int64_t(1) << 32);
  const bool vec = aligned(Wq, 4) && (K & 3) == 0;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    int64_t row, g;
    split_index(i, words, small, row, g);
    const int64_t k0 = g * 20;
    const int8_t* wr = Wq + row * K;
    uint32_t d[20];
    if (vec && k0 + 20 <= K) {
#pragma unroll
      for (int v = 0; v < 5; ++v) {
        const char4 c = reinterpret_cast<const char4*>(wr + k0)[v];
        d[4 * v + 0] = uint32_t(c.x + 1);
        d[4 * v + 1] = uint32_t(c.y + 1);
        d[4 * v + 2] = uint32_t(c.z + 1);
        d[4 * v + 3] = uint32_t(c.w + 1);
      }
    } else {
#pragma unroll
      for (int k = 0; k < 20; ++k) d[k] = (k0 + k < K) ? uint32_t(wr[k0 + k] + 1) : 1u;
    }
    uint32_t word = 0u;
#pragma unroll
    for (int b = 0; b < 4; ++b)
      word |= pack5_digits(d[5 * b], d[5 * b + 1], d[5 * b + 2], d[5 * b + 3], d[5 * b + 4]) << (8 * b);
    *reinterpret_cast<uint32_t*>(Wp + row * ldp + 4 * g) = word;
  }
}

// Wp [N,ldp] -> Wq [N,ldq] int8, the first K trits of each row.  One thread per
// packed byte.
__global__ void __launch_bounds__(256)
unpack5_kernel(const uint8_t* __restrict__ Wp, int64_t N, int64_t K, int64_t ldp,
               int8_t* __restrict__ Wq, int64_t ldq) {
  const int64_t nb = ceil_div(K, 5);
  const int64_t total = N * nb;
  const bool small = total < (int64_t(1) << 32);
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    int64_t row, j;
    split_index(i, nb, small, row, j);
    const uint32_t b = Wp[row * ldp + j];
    int8_t* out = Wq + row * ldq + 5 * j;
    int t5[5];
    unpack5_byte(b, t5);
#pragma unroll
    for (int k = 0; k < 5; ++k)
      if (5 * j + k < K) out[k] = int8_t(t5[k]);
  }
}

}  // namespace bl
