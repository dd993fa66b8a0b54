// Decoding packed trits: the per-lane table of the first four trits of a byte,
// the fifth trit computed four bytes at a time, and the decode order of the
// activations that pairs with them.
//
// Packing of "ultragraph-1bit 0.12.0" (PyPI), section "A whole ternary GPT"
// (bit-packed ternary bytes), as this library stores it: byte j of a row holds
// trits 5j..5j+4 as b = sum_k (t_k + 1) 3^k, so digit d_k = floor(b/3^k) mod 3
// and t_k = d_k - 1.  Bytes above 242 are not codes.
//
// Decode order.  For packed word g of a row (bytes 4g..4g+3, trits 20g..20g+19)
// the decoders produce five 32-bit words of int8 trits:
//   word i < 4:  t0..t3 of byte 4g+i          (trits 5(4g+i) .. 5(4g+i)+3)
//   word 4:      t4 of bytes 4g..4g+3          (trits 5(4g+i)+4, i = 0..3)
// The activation codes are laid out in the same order (trit k of the row sits
// at position dorder_pos(k)), so every dot product pairs the right codes and no
// byte of a decoded word has to move.
#pragma once

#include <cstdint>

namespace bl {

constexpr uint32_t kLutBytes = 256 * 256;   // a row for every byte value: no read leaves the table

// The table as it sits in shared memory: word b*64 + l (l < 32) holds trits
// t0..t3 of byte b as four int8 (lane l's copy; words 32..63 of a row repeat
// them, so the row pitch is 256 bytes and one byte_perm forms an address).
// Bytes above 242 read as 121 (four zero trits).  Each CTA writes it with 16
// stores of 16 bytes per 256-byte row (no global traffic).
__device__ __forceinline__ uint32_t trit_word(uint32_t b) {
  uint32_t x = b > 242u ? 121u : b, v = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t q = x / 3u;
    v |= ((x - 3u * q + 255u) & 0xFFu) << (8 * k);
    x = q;
  }
  return v;
}
// The same table as a compile-time constant in global memory, for CTAs that
// copy it (one bulk copy) instead of writing it.
struct TritLut {
  uint32_t w[256 * 64];
};
constexpr TritLut make_trit_lut() {
  TritLut t{};
  for (uint32_t b = 0; b < 256; ++b) {
    uint32_t x = b > 242u ? 121u : b, v = 0;
    for (int k = 0; k < 4; ++k) {
      v |= ((x % 3u + 255u) & 0xFFu) << (8 * k);
      x /= 3u;
    }
    for (uint32_t l = 0; l < 64; ++l) t.w[b * 64 + l] = v;
  }
  return t;
}
__device__ __align__(128) const TritLut g_trit_lut = make_trit_lut();

// Threads tid = 0 .. nthreads-1 of the CTA write the table at `lut` (kLutBytes,
// 16-byte aligned); the caller's next CTA barrier makes it visible.
__device__ __forceinline__ void build_trit_lut(unsigned char* lut, int tid, int nthreads) {
  for (int i = tid; i < 256 * 16; i += nthreads) {
    const uint32_t v = trit_word(uint32_t(i) >> 4);
    *reinterpret_cast<uint4*>(lut + 16 * i) = make_uint4(v, v, v, v);
  }
}

// Trits t0..t3 of byte `bb` (0..3) of packed word w, from the table at `lut`
// (shared memory); lanebase = 4 * lane.
__device__ __forceinline__ uint32_t lut_t0123(const unsigned char* lut, uint32_t w, uint32_t lanebase, int bb) {
  return *reinterpret_cast<const uint32_t*>(lut + __byte_perm(w, lanebase, 0x5504u | (uint32_t(bb) << 4)));
}

// 64 * d4 of the four bytes of w, one per byte: b * 203 in 16-bit lanes holds
// floor(b/81) in bits 14..15 for every b <= 242 (203 / 2^14 lies between 1/81
// and 1/81 + 1/(81 * 243)), and a byte_perm gathers those bytes.
__device__ __forceinline__ uint32_t d4x64(uint32_t w) {
  const uint32_t E = __byte_perm(w, 0u, 0x4240u) * 203u;
  const uint32_t O = __byte_perm(w, 0u, 0x4341u) * 203u;
  return __byte_perm(E, O, 0x7351u) & 0xC0C0C0C0u;
}

// t4 = d4 - 1 of the four bytes of w as four int8.
__device__ __forceinline__ uint32_t t4_word(uint32_t w) {
  return ((d4x64(w) >> 6) + 0x7F7F7F7Fu) ^ 0x80808080u;
}

// Position of trit k of a row in the decode order.
__host__ __device__ __forceinline__ uint32_t dorder_pos(uint32_t k) {
  const uint32_t j = k / 5u, r = k - 5u * j;
  return 20u * (j >> 2) + (r < 4u ? 4u * (j & 3u) + r : 16u + (j & 3u));
}

// Length of a row in the decode order: whole packed words.
__host__ __device__ constexpr int64_t dorder_len(int64_t K) { return 20 * ((K + 19) / 20); }

}  // namespace bl
