// Deployed checkpoint of BitLinear layers: file writer and reader.
//
// "ultragraph-1bit 0.12.0" (PyPI), section "A whole ternary GPT": the deployed
// checkpoint stores the ternary weights at five per byte (about 1.6 bits each)
// plus the small float32 pieces, and a model loaded from it runs straight from
// the stored bytes with outputs identical to the model that wrote it.  Layout
// (little-endian, no padding):
//
//   header := "BLT5"  version:u32 = 1  count:u32  reserved:u32 = 0
//   layer  := name_len:u32 (<= 255)  name bytes
//             N:u64  K:u64  flags:u32 (bit 0: bias follows)  beta:u32 (float32 bits)
//             packed rows: N * ceil(K/5) bytes (the BL_W_PACK5 rows without
//             their padding to 16 bytes)
//             [bias: N float32]
//
// Host code only: the device buffers move with cudaMemcpy2D / cudaMemcpy
// (synchronous), through host staging buffers of at most kIoChunk bytes.
#pragma once

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include <cuda_runtime.h>

#include "bitlinear.h"
#include "common.cuh"

namespace bl {
namespace io {

constexpr char kMagic[4] = {'B', 'L', 'T', '5'};
constexpr uint32_t kVersion = 1;
constexpr size_t kIoChunk = size_t(64) << 20;
constexpr uint32_t kMaxName = 255;

inline void put_u32(unsigned char* p, uint32_t v) {
  for (int i = 0; i < 4; ++i) p[i] = (unsigned char)(v >> (8 * i));
}
inline void put_u64(unsigned char* p, uint64_t v) {
  for (int i = 0; i < 8; ++i) p[i] = (unsigned char)(v >> (8 * i));
}
inline uint32_t get_u32(const unsigned char* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; ++i) v |= uint32_t(p[i]) << (8 * i);
  return v;
}
inline uint64_t get_u64(const unsigned char* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; ++i) v |= uint64_t(p[i]) << (8 * i);
  return v;
}

// A layer record's fixed fields, as read from a file.
struct Record {
  char name[kMaxName + 1];
  uint64_t N, K;
  uint32_t flags, beta_bits;
  long packed_off;   // file offset of the packed rows
};

struct File {
  FILE* f = nullptr;
  ~File() {
    if (f) fclose(f);
  }
};

// Reads one layer record's fixed part at the current position and leaves the
// file at the start of the next record; false on a malformed or short file.
inline bool read_record(FILE* f, Record& r) {
  unsigned char b[4];
  if (fread(b, 1, 4, f) != 4) return false;
  const uint32_t nlen = get_u32(b);
  if (nlen > kMaxName) return false;
  if (nlen && fread(r.name, 1, nlen, f) != nlen) return false;
  r.name[nlen] = '\0';
  unsigned char h[24];
  if (fread(h, 1, 24, f) != 24) return false;
  r.N = get_u64(h);
  r.K = get_u64(h + 8);
  r.flags = get_u32(h + 16);
  r.beta_bits = get_u32(h + 20);
  if (r.N < 1 || r.K < 1 || r.N > (uint64_t(1) << 40) || r.K > uint64_t(kMaxK) || (r.flags & ~1u)) return false;
  r.packed_off = ftell(f);
  const uint64_t cb = (r.K + 4) / 5;
  const uint64_t skip = r.N * cb + ((r.flags & 1u) ? 4 * r.N : 0);
  if (fseek(f, long(skip), SEEK_CUR) != 0) return false;
  return true;
}

// Opens `path`, checks the header and returns the layer count (-1 on error).
inline int open_checked(const char* path, File& file) {
  if (!path) return -1;
  file.f = fopen(path, "rb");
  if (!file.f) return -1;
  unsigned char h[16];
  if (fread(h, 1, 16, file.f) != 16 || memcmp(h, kMagic, 4) != 0 || get_u32(h + 4) != kVersion) return -1;
  const uint32_t count = get_u32(h + 8);
  return count > 0x7fffffffu ? -1 : int(count);
}

// Positions `file` on layer `index` (reading every record before it); the
// record of that layer lands in `r`.  False on error or a short file.
inline bool seek_layer(File& file, int index, Record& r) {
  for (int i = 0; i <= index; ++i)
    if (!read_record(file.f, r)) return false;
  return true;
}

}  // namespace io
}  // namespace bl
