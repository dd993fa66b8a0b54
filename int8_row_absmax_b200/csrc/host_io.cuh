// Moving a step's activations in from host memory without the copy engine.
//
// A decode step's inputs are a few tens of KB.  A host-to-device copy by the
// copy engine between two kernels costs far more than its bytes (the stream
// hands work from the compute engine to the copy engine and back), so for
// page-locked host memory that is mapped into the device's address space the
// library reads the rows with a kernel of its own: plain loads over the bus,
// all issued before the kernel waits for the previous grid on the stream (the
// loads' round trip overlaps that grid's tail), stores into the device staging
// buffers after the wait (the previous grid may still read them).
#pragma once

#include <cstdint>

#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kSpanMax = 8;          // spans per launch
constexpr int kSpanThreads = 256;
constexpr int kSpanPre = 4;          // units each thread loads before the wait

// Up to kSpanMax copies of whole units (16 bytes when every span allows it,
// else 4): span i covers global units [first[i], first[i+1]).
struct SpanCopy {
  char* dst[kSpanMax];
  const char* src[kSpanMax];
  int64_t first[kSpanMax + 1];
  int n;
};

template <int kUnit>
__device__ __forceinline__ void span_locate(const SpanCopy& a, int64_t g, char*& d, const char*& s) {
  int i = 0;
#pragma unroll
  for (int j = 1; j < kSpanMax; ++j)
    if (j < a.n && g >= a.first[j]) i = j;
  const int64_t off = (g - a.first[i]) * kUnit;
  d = a.dst[i] + off;
  s = a.src[i] + off;
}

template <int kUnit>
struct SpanWord;
template <>
struct SpanWord<16> {
  using T = uint4;
};
template <>
struct SpanWord<4> {
  using T = uint32_t;
};

// Grid-stride over the units; the first kSpanPre rounds are loaded before the
// dependency wait and stored after it.
template <int kUnit>
__global__ void __launch_bounds__(kSpanThreads) span_copy_kernel(const __grid_constant__ SpanCopy a) {
  using T = typename SpanWord<kUnit>::T;
  griddep_launch_dependents();
  const int64_t total = a.first[a.n];
  const int64_t stride = int64_t(gridDim.x) * kSpanThreads;
  const int64_t g0 = int64_t(blockIdx.x) * kSpanThreads + threadIdx.x;
  T v[kSpanPre];
#pragma unroll
  for (int r = 0; r < kSpanPre; ++r) {
    const int64_t g = g0 + r * stride;
    if (g < total) {
      char* d;
      const char* s;
      span_locate<kUnit>(a, g, d, s);
      v[r] = *reinterpret_cast<const T*>(s);
    }
  }
  griddep_wait();
#pragma unroll
  for (int r = 0; r < kSpanPre; ++r) {
    const int64_t g = g0 + r * stride;
    if (g < total) {
      char* d;
      const char* s;
      span_locate<kUnit>(a, g, d, s);
      *reinterpret_cast<T*>(d) = v[r];
    }
  }
  for (int64_t g = g0 + kSpanPre * stride; g < total; g += stride) {
    char* d;
    const char* s;
    span_locate<kUnit>(a, g, d, s);
    *reinterpret_cast<T*>(d) = *reinterpret_cast<const T*>(s);
  }
}

}  // namespace bl
