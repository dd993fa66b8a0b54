// Absmean ternarization in one pass over W, one cooperative launch.
//
// "ultragraph -- when the graph is the 1-bit LLM, part 2", section "the bytes":
//   beta = (1/n) sum_i |W_i| + eps,   W_q = clip(round(W / beta), -1, 1).
//
// beta is a mean over the whole tensor, so no code is final before every weight
// has been read, and the two-pass form (absmean_kernel, then a ternarize kernel)
// reads W from HBM twice.  wquant_kernel reads it once.  One CTA per SM, all
// resident together (cooperative launch):
//
//   0. chunks of W (512 groups of 20 weights, one contiguous range) are handed
//      out in a strided order, so the first chunk of every CTA is spread evenly
//      over the tensor.  Each CTA's first chunk is its share of the sample: its
//      mean |w| goes to the workspace; grid barrier A.  Every CTA turns the
//      sample into the same band [T_lo, T_hi] that holds the ternary threshold
//      T of the exact beta with overwhelming probability (7 standard errors of
//      the mean plus a 1e-4 relative margin);
//   1. W streams once (bulk copies into a ring of shared-memory stages, chunks
//      handed out dynamically).  Every weight's magnitude is added in float64,
//      and each 20-weight group is coded against T_hi at once: |w| >= T_hi gives
//      +-1, anything else 0; a group holding a weight with T_lo <= |w| < T_hi has
//      its index appended to the warp's list.  At grid barrier B (all CTAs
//      have added their float64 sums) every CTA certifies beta from the same
//      total: T is within E = (L + 4) 2^-52 T of the exact sum (L = the
//      longest chain of float64 additions, all addends being non-negative), and
//      beta = float32(float64(S) / n) + eps is monotone in S, so when T - E and
//      T + E give the same beta that is the exact beta.  Otherwise (a mean
//      within about 1e-13 of a float32 rounding boundary, or a non-finite sum)
//      every CTA adds the magnitudes again exactly, as integers in units of
//      2^-149 (the absmean_kernel method), and the last one rounds the exact
//      total.  With beta and T known: mode 0 if T_lo <= T <= T_hi and no list
//      overflowed, else mode 1;
//   2. mode 0: each warp re-codes the groups on its list from W against T;
//      mode 1: the grid re-ternarizes the whole tensor.
//
// Weights with |w| < T_lo are below T, those with |w| >= T_hi are at or above
// it, and every group with a weight in between is redone against T, so the
// codes equal those of the two-pass kernels (and of the IEEE division) for any
// input; the sample only decides how much work phase 2 has.  Every wait is
// bounded: a barrier that times out records kDevTimeout and forces mode 1.
//
// The BitLinear forward for M <= 4 rows of X (decode) rides on the same pass
// (kM > 0): while phase 0 waits, every CTA quantizes X (per-row absmax, the
// codes of bl_quantize_act) into shared memory as small integer floats; in
// phase 1 each group adds sum_k t_k x_q[k] (exact in float32: |sum| <= 20*127)
// into int32 row accumulators (a row-segmented warp reduction, one atomic per
// segment); phase 2 adds, for every re-coded group, the exact difference
// between its final and provisional codes; the CTA that leaves last writes
// Y = float(acc) (s beta) [+ b] and clears the accumulators.
#pragma once

#include "act_quant.cuh"
#include "weight_quant.cuh"

namespace bl {

constexpr int kFuGroups = kAbsConsumers;               // 20-weight groups per chunk, one per thread
constexpr int kFuStageFloats = kFuGroups * 20;         // 10240 floats
constexpr uint32_t kFuStageBytes = kFuStageFloats * 4; // 40 KB
constexpr int kFuStages = 5;                           // 200 KB in flight per SM
constexpr int kFuStagesFwd = 4;                        // with the forward: room for X codes
constexpr int kFuPreStages = 2;                        // issued before the band is known
constexpr int kFwdMaxM = 4;
constexpr uint32_t kFwdXBytesMax = 48 * 1024;          // float X codes in shared memory
constexpr int kFuSmem = kFuStages * int(kFuStageBytes);
constexpr int kFuWarps = kAbsConsumers / 32;           // lists per CTA
constexpr int64_t kFusedMinN = int64_t(1) << 20;       // smaller tensors take the two-pass path
constexpr double kBandSigmas = 7.0;
constexpr double kBandRelMargin = 1e-4;
constexpr size_t kFuListOff = kAbsWsBytes;             // lists follow the accumulator block

// List capacity per warp: 1/8 of the groups a warp streams on average, + 16.
__host__ __device__ inline int64_t fused_cap_w(int64_t ngroups, int grid) {
  const int64_t warps = int64_t(grid) * kFuWarps;
  return 16 + ((ngroups + warps - 1) / warps + 7) / 8;
}

// Workspace bytes for any grid up to kAbsMaxCtas CTAs (8-byte list entries):
// grid*16*cap_w <= grid*16*(18 + ngroups/(grid*128)) <= 288*kAbsMaxCtas + ngroups/8.
// With the forward (M rows), int32 row accumulators [M, N] come first.
__host__ __device__ inline size_t fused_acc_bytes(int64_t M, int64_t N) {
  return (size_t(M) * size_t(N) * 4 + 255) & ~size_t(255);
}
__host__ __device__ inline size_t fused_ws_bytes(int64_t N, int64_t K, int64_t M = 0) {
  const int64_t ngroups = N * ((K + 19) / 20);
  const size_t entries = size_t(288) * kAbsMaxCtas + size_t(ngroups / 8 + 1);
  return (kFuListOff + fused_acc_bytes(M, N) + entries * 8 + 255) & ~size_t(255);
}

struct WqArgs {
  const float* W;
  int64_t N, K;
  float eps;
  void* out;                       // packed [N, ldo] or int8 [N, ldo = K]
  int64_t ldo;
  AbsAccum* acc;                   // accumulator block (workspace start)
  unsigned long long* list;        // per-warp lists of groups to re-code
  int cap_w;
  uint32_t stride, gpr_magic;
  float* beta_out;
  // the forward (kM > 0)
  const float* X;                  // [M, K] float32, 16-byte aligned
  const float* bias;               // [N] or nullptr
  float* Y;                        // [M, N]
  int* yacc;                       // [M, N] int32 row sums (cleared in phase 0)
  uint32_t xf_off;                 // shared-memory offset of the X codes
};

// A chunk order whose first `grid` entries are spread over the tensor: handout
// i takes chunk (i * stride) mod nch, stride ~ nch / grid and coprime to nch.
inline uint32_t chunk_stride(int64_t nch, int grid) {
  auto gcd = [](int64_t a, int64_t b) {
    while (b) {
      const int64_t t = a % b;
      a = b;
      b = t;
    }
    return a;
  };
  int64_t s = nch / (grid > 0 ? grid : 1);
  if (s < 1) s = 1;
  while (gcd(s, nch) != 1) ++s;
  return uint32_t(s);
}

struct TernBand {
  uint32_t lo, hi;  // float bits of T_lo, T_hi (non-negative floats order as integers)
  int ok;
};

// The band from the sample: mean and standard error over the sampled chunk
// means; the beta interval is rounded outwards through the float32 rounding and
// the +eps, and mapped through the (monotone) threshold function.
__device__ inline TernBand ternary_band(double s1, double s2, double units, float eps) {
  TernBand b;
  b.lo = 0u;
  b.hi = 0u;
  b.ok = 0;
  if (!(units >= 2.0)) return b;
  const double mu = s1 / units;
  double var = (s2 - s1 * mu) / (units - 1.0);
  if (!(var > 0.0)) var = 0.0;
  const double h = kBandSigmas * sqrt(var / units) + kBandRelMargin * mu;
  if (!(mu >= 0.0 && mu < 1e38 && h >= 0.0 && h < 1e38)) return b;
  const double mlo = mu - h > 0.0 ? mu - h : 0.0;
  const float blo = __fadd_rd(__double2float_rd(mlo), eps);
  const float bhi = __fadd_ru(__double2float_ru(mu + h), eps);
  if (!(bhi < 1.0e38f) || !(blo >= 0.f)) return b;
  b.lo = __float_as_uint(ternary_threshold(blo));
  b.hi = __float_as_uint(ternary_threshold(bhi));
  // the step tests below need both thresholds' predecessors to have biased
  // exponents >= 24 (then 2^(151-e) is a float)
  b.ok = ((b.lo - 1u) >> 23) >= 24u && b.hi < 0x7F800000u;
  return b;
}

// [x >= T] as 0.0 / 1.0 from the predecessor Tp of T: for floats x > Tp the
// rounded x - Tp is at least ulp(Tp), which the scale 2^(151 - e(Tp)) lifts to
// >= 2, and the saturating multiply clamps to [0, 1] (NaN to 0).  Two
// floating-point instructions instead of an integer compare and select.
struct StepConst {
  float tp;     // predecessor of T
  float scale;  // 2^(151 - biased exponent of tp)
};
__device__ inline StepConst step_const(uint32_t tbits) {
  StepConst c;
  const uint32_t pb = tbits - 1u;
  c.tp = __uint_as_float(pb);
  c.scale = __uint_as_float((278u - (pb >> 23)) << 23);
  return c;
}
__device__ __forceinline__ float mul_sat(float a, float b) {
  float d;
  asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}
__device__ __forceinline__ float step_ge(float ax, StepConst c) {
  return mul_sat(__fsub_rn(ax, c.tp), c.scale);
}

__device__ __forceinline__ float f4get(const float4& v, int j) {
  return j == 0 ? v.x : (j == 1 ? v.y : (j == 2 ? v.z : v.w));
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const unsigned int* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned int* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// Bounded wait for *p >= target; false after kWaitLimitNs.
__device__ inline bool wait_u32_geq(const unsigned int* p, uint32_t target) {
  if (ld_acquire_u32(p) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_u32(p) < target) {
    __nanosleep(20);
    if (globaltimer_ns() - t0 > kWaitLimitNs) return false;
  }
  return true;
}

// The sample's sums over all CTAs in one fixed order (every CTA computes
// bit-identical values), then the band.  One whole warp; result in lane 0.
__device__ inline TernBand band_from_parts(const AbsAccum* acc, int nparts, float eps, int lane) {
  double a = 0.0, b = 0.0, c = 0.0;
  for (int i = lane; i < nparts; i += 32) {
    const double m = __ldcg(&acc->est_part[i][0]);
    if (m >= 0.0) {
      a += m;
      b += __ldcg(&acc->est_part[i][1]);
      c += 1.0;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_down_sync(0xffffffffu, a, o);
    b += __shfl_down_sync(0xffffffffu, b, o);
    c += __shfl_down_sync(0xffffffffu, c, o);
  }
  return ternary_band(a, b, c, eps);
}

// beta for every exact sum S with |S - T| <= E, or NaN when the interval
// straddles a rounding boundary (or T is not a finite non-negative number).
__device__ inline float certified_beta(double T, double E, int64_t n, float eps) {
  if (!(T >= 0.0 && T <= 1.0e300 && E >= 0.0)) return __int_as_float(0x7FC00000);
  double lo = __dsub_rd(T, E);
  if (lo < 0.0) lo = 0.0;
  const double hi = __dadd_ru(T, E);
  const float b_lo = __fadd_rn(__double2float_rn(__ddiv_rn(lo, double(n))), eps);
  const float b_hi = __fadd_rn(__double2float_rn(__ddiv_rn(hi, double(n))), eps);
  return b_lo == b_hi ? b_lo : __int_as_float(0x7FC00000);
}

// beta from the exact pass's limb totals (three 32-bit limbs, units 2^(kFastLo-150)).
__device__ inline float beta_from_limbs(unsigned long long L0, unsigned long long L1,
                                        unsigned long long L2, int64_t n, float eps) {
  unsigned long long lo64 = L0 + (L1 << 32);
  const unsigned long long hi64 = (L1 >> 32) + L2 + (lo64 < L0 ? 1ull : 0ull);
  double D;
  if (hi64 == 0ull) {
    D = ldexp(__ull2double_rn(lo64), int(kFastLo) - 150);
  } else {
    const int sh = 64 - __clzll(hi64);           // drop sh low bits, keep a sticky bit
    unsigned long long top = (hi64 << (64 - sh)) | (lo64 >> sh);
    top |= (lo64 << (64 - sh)) != 0ull ? 1ull : 0ull;
    D = ldexp(__ull2double_rn(top), sh + int(kFastLo) - 150);
  }
  return __fadd_rn(__double2float_rn(__ddiv_rn(D, double(n))), eps);
}

// [x >= T] for the step constants c, with the sign of x: -1, 0 or +1 as a float.
__device__ __forceinline__ float signed_step(float x, StepConst c) {
  return __uint_as_float(__float_as_uint(step_ge(fabsf(x), c)) | (__float_as_uint(x) & 0x80000000u));
}

// The code of bl_quantize_act as a float (-127 .. 127); `tie` as in act_code_try.
__device__ __forceinline__ float act_codef_try(float x, float r, bool& tie) {
  const float y = fminf(fmaxf(__fmul_rn(x, r), -float(kActQmax)), float(kActQmax));
  const float q = __fsub_rn(__fadd_rn(y, 12582912.0f), 12582912.0f);
  tie |= fabsf(fabsf(__fsub_rn(y, q)) - 0.5f) < 3.0517578125e-05f;
  return q;
}

// Adds v into yacc[m * N + key] once per run of equal keys among the warp's
// lanes (keys of one warp are non-decreasing; key -1: nothing).
__device__ __forceinline__ void add_by_row(int* yacc, int64_t idx_base, int key, int v, int lane) {
  if (__shfl_sync(0xffffffffu, key, 0) == __shfl_sync(0xffffffffu, key, 31)) {  // one row: the usual case
    const int t = __reduce_add_sync(0xffffffffu, v);
    if (lane == 0 && key >= 0 && t != 0) atomicAdd(yacc + idx_base + key, t);
    return;
  }
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const int vv = __shfl_down_sync(0xffffffffu, v, d);
    const int kk = __shfl_down_sync(0xffffffffu, key, d);
    if (lane + d < 32 && kk == key) v += vv;
  }
  const int kp = __shfl_up_sync(0xffffffffu, key, 1);
  if (key >= 0 && (lane == 0 || kp != key) && v != 0) atomicAdd(yacc + idx_base + key, v);
}

// Chunks are 512 consecutive 20-weight groups in row-major group order (a group
// never crosses a row, so a chunk is one contiguous range of W); consumer thread
// t takes group t of every chunk: five 128-bit shared-memory loads, 20 weights,
// one output word.  list: per warp, cap_w 8-byte entries (row << 32 | group).
template <bool kPacked, int kM>
__global__ void __launch_bounds__(kAbsThreads, 1)
wquant_kernel(const __grid_constant__ WqArgs a) {
  constexpr int kStages = kM > 0 ? kFuStagesFwd : kFuStages;
  constexpr int kMM = kM > 0 ? kM : 1;
  extern __shared__ __align__(128) unsigned char stage_smem[];
  __shared__ uint64_t full[kStages], empty[kStages];
  __shared__ long long s_row0[kStages];
  __shared__ int s_g0[kStages], s_ng[kStages];
  __shared__ int s_issued[kStages];
  __shared__ unsigned long long s_bins[256];
  __shared__ unsigned long long s_limb[3];
  __shared__ unsigned long long s_word[kBigWords + 3];
  __shared__ uint32_t s_big[kBigWords];
  __shared__ int s_flag;
  __shared__ int s_timeout;
  __shared__ unsigned long long s_binv[255];
  __shared__ unsigned long long s_wsum[3 * (kAbsThreads / 32)];
  __shared__ double s_dpart[kAbsThreads / 32];
  __shared__ float s_samp[kFuWarps];
  __shared__ int s_scnt[kFuWarps];
  __shared__ float s_xred[kMM][kFuWarps];
  __shared__ float s_xs[kMM];
  __shared__ bool s_last;
  __shared__ TernBand s_band;
  __shared__ int s_mode, s_next;
  __shared__ float s_beta;
  const float* __restrict__ W = a.W;
  const int64_t N = a.N, K = a.K, ldo = a.ldo;
  const float eps = a.eps;
  void* __restrict__ out = a.out;
  AbsAccum* __restrict__ acc = a.acc;
  const int cap_w = a.cap_w;
  float* __restrict__ beta_out = a.beta_out;
  const float* xf = reinterpret_cast<const float*>(stage_smem + a.xf_off);  // kM > 0 only
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  for (int i = tid; i < 256; i += blockDim.x) s_bins[i] = 0ull;
  const int64_t gpr = ceil_div(K, 20);             // output words (groups) per row, <= 6554
  const int64_t ngroups = N * gpr;
  const int64_t nch = ceil_div(ngroups, kFuGroups);
  const int64_t n = N * K;
  const int n_static = nch >= 2 * int64_t(gridDim.x) ? int(nch / gridDim.x) - 1 : 0;
  // q / gpr for q < gpr + 512: hi32(q * ceil(2^32 / gpr)) is exact while q * gpr < 2^32
  auto div_gpr = [&](uint32_t q) -> uint32_t { return gpr == 1 ? q : __umulhi(q, a.gpr_magic); };
  if (tid == 0) {
    s_timeout = 0;
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFuWarps);
      s_issued[s] = 0;
    }
    fence_mbar_init();
  }
  __syncthreads();

  double da0 = 0.0, da1 = 0.0;                      // this thread's float64 sums of |w|
  int wcount = 0;                                   // this warp's list length
  unsigned long long* wl = a.list + int64_t(blockIdx.x * kFuWarps + (warp < kFuWarps ? warp : 0)) * cap_w;
  if (warp == kFuWarps) {
    // producer warp: lane 0 hands out chunks and issues the copies; only the
    // first kFuPreStages go out before the band is known, so the first chunk
    // and barrier A do not queue behind a full ring's worth of copies.
    // Handouts: this CTA's first n_static are blockIdx.x + k * grid (so its
    // first one is its share of the stratified sample), the tail comes from a
    // counter whose next value is always requested one handout ahead.
    unsigned int tail = 0u;
    bool more = true;
    auto issue = [&](int it) -> bool {   // false: stop marker sent, or a wait gave up
      const int s = it % kStages;
      if (it >= kStages && !mbar_wait(&empty[s], uint32_t(it / kStages - 1) & 1u)) {
        s_timeout = 1;
        return false;
      }
      int64_t h;
      if (it < n_static) {
        h = int64_t(blockIdx.x) + int64_t(it) * gridDim.x;
      } else {
        h = int64_t(n_static) * gridDim.x + tail;
        if (h < nch) tail = atomicAdd(&acc->next_chunk, 1u);
      }
      if (h >= nch) {
        s_ng[s] = -1;
        s_issued[s] += 1;
        mbar_arrive(&full[s]);
        return false;
      }
      const int64_t chunk = int64_t((static_cast<unsigned long long>(h) * a.stride) % uint64_t(nch));
      const int64_t G0 = chunk * kFuGroups;
      const int64_t G1 = min(ngroups, G0 + kFuGroups);
      const int64_t row0 = G0 / gpr, g0 = G0 - row0 * gpr;
      const int64_t rowL = (G1 - 1) / gpr, gL = (G1 - 1) - rowL * gpr;
      const int64_t f0 = row0 * K + 20 * g0;                    // multiples of 4 floats
      const int64_t f1 = rowL * K + min(K, 20 * gL + 20);
      const uint32_t bytes = uint32_t((f1 - f0) * 4);           // <= 40 KB, % 16 == 0
      s_row0[s] = row0;
      s_g0[s] = int(g0);
      s_ng[s] = int(G1 - G0);
      s_issued[s] += 1;
      fence_proxy_async_smem();
      mbar_arrive_expect_tx(&full[s], bytes);
      bulk_g2s(stage_smem + size_t(s) * kFuStageBytes, W + f0, bytes, &full[s]);
      return true;
    };
    int it = 0;
    if (lane == 0) {
      tail = atomicAdd(&acc->next_chunk, 1u);
      for (; it < kFuPreStages && more; ++it) more = issue(it);
    }
    __syncwarp();
    named_bar_sync(3, kAbsThreads);                  // the consumers have the band
    if (lane == 0)
      for (; more; ++it) more = issue(it);
  } else {
    // ---- phase 0: X codes (forward), then this CTA's sample and barrier A ----
    if constexpr (kM > 0) {
      // the row sums start at zero: cleared here, before barrier A, so every
      // CTA's clearing is visible before any CTA adds into them
      for (int64_t i = int64_t(blockIdx.x) * kAbsConsumers + tid; i < int64_t(kM) * N;
           i += int64_t(gridDim.x) * kAbsConsumers)
        a.yacc[i] = 0;
      float* xw = reinterpret_cast<float*>(stage_smem + a.xf_off);
      const int K4 = int(K >> 2);                    // K % 4 == 0, X 16-byte aligned
      bool badx = false;
#pragma unroll
      for (int m = 0; m < kM; ++m) {
        const float4* xr = reinterpret_cast<const float4*>(a.X + int64_t(m) * K);
        float mx = 0.f;
        for (int i = tid; i < K4; i += kAbsConsumers) {
          const float4 v = __ldg(xr + i);
          const float t = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
          badx |= !(t <= 3.402823466e38f) | (v.x != v.x) | (v.y != v.y) | (v.z != v.z) | (v.w != v.w);
          mx = fmaxf(mx, t);
        }
        mx = warp_max(mx);
        if (lane == 0) s_xred[m][warp] = mx;
      }
      if (badx) raise_status(kDevNonFinite);
      named_bar_sync(1, kAbsConsumers);
#pragma unroll
      for (int m = 0; m < kM; ++m) {
        const float w = warp_max(lane < kFuWarps ? s_xred[m][lane] : 0.f);
        const float sc = __fadd_rn(__fdiv_rn(w, float(kActQmax)), eps);
        const float rc = act_recip(sc);
        if (tid == 0) s_xs[m] = sc;
        const float4* xr = reinterpret_cast<const float4*>(a.X + int64_t(m) * K);
        float4* xo = reinterpret_cast<float4*>(xw + int64_t(m) * K);
        for (int i = tid; i < K4; i += kAbsConsumers) {
          const float4 v = __ldg(xr + i);
          bool tie = rc == 0.f;
          float4 q;
          q.x = act_codef_try(v.x, rc, tie);
          q.y = act_codef_try(v.y, rc, tie);
          q.z = act_codef_try(v.z, rc, tie);
          q.w = act_codef_try(v.w, rc, tie);
          if (tie) {   // rare: a quotient near a half-integer; exact division for those elements
            if (act_near_tie(v.x, rc)) q.x = float(act_code_slow(v.x, sc));
            if (act_near_tie(v.y, rc)) q.y = float(act_code_slow(v.y, sc));
            if (act_near_tie(v.z, rc)) q.z = float(act_code_slow(v.z, sc));
            if (act_near_tie(v.w, rc)) q.w = float(act_code_slow(v.w, sc));
          }
          xo[i] = q;
        }
      }
    }
    {
      float sa = 0.f;
      int cnt = 0;
      if (mbar_wait(&full[0], 0u)) {
        const int ng = s_ng[0];
        if (tid < ng) {
          const uint32_t q = uint32_t(s_g0[0]) + uint32_t(tid);
          const uint32_t dr = div_gpr(q);
          const int g = int(q - dr * uint32_t(gpr));
          cnt = int(min(int64_t(20), K - 20 * int64_t(g)));
          const float* gs = reinterpret_cast<const float*>(stage_smem) + (int(dr) * int(K) + 20 * (g - s_g0[0]));
          for (int k = 0; k < cnt; ++k) sa += fabsf(gs[k]);
        }
      } else {
        s_timeout = 1;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        sa += __shfl_xor_sync(0xffffffffu, sa, o);
        cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
      }
      if (lane == 0) {
        s_samp[warp] = sa;
        s_scnt[warp] = cnt;
      }
      named_bar_sync(1, kAbsConsumers);
      if (tid == 0) {
        double ssum = 0.0;
        int64_t sc = 0;
        for (int w = 0; w < kFuWarps; ++w) {
          ssum += double(s_samp[w]);
          sc += s_scnt[w];
        }
        const double m = sc > 0 ? ssum / double(sc) : -1.0;
        acc->est_part[blockIdx.x][0] = m;
        acc->est_part[blockIdx.x][1] = m * m;
        __threadfence();
        atomicAdd(&acc->bar_a, 1u);
        if (!wait_u32_geq(&acc->bar_a, gridDim.x)) {
          raise_status(kDevTimeout);
          atomicOr(&acc->overflow, 2u);    // bands may differ between CTAs: force mode 1
        }
      }
      named_bar_sync(1, kAbsConsumers);
      if (warp == 1) {
        const TernBand bd = band_from_parts(acc, int(gridDim.x), eps, lane);
        if (lane == 0) s_band = bd;
      }
      named_bar_sync(3, kAbsThreads);                // band out; the producer goes on
    }

    // ---- phase 1: stream W, float64 sum, codes against T_hi, band lists ----
    // an unusable band codes everything 0 (mode 1 then redoes the tensor)
    const StepConst sc_hi = s_band.ok ? step_const(s_band.hi) : StepConst{__int_as_float(0x7F800000), 1.f};
    const StepConst sc_lo = s_band.ok ? step_const(s_band.lo) : StepConst{__int_as_float(0x7F800000), 1.f};
    for (int it = 0;; ++it) {
      const int s = it % kStages;
      if (!mbar_wait(&full[s], uint32_t(it / kStages) & 1u)) {
        s_timeout = 1;
        break;
      }
      const int ng = s_ng[s];
      if (ng < 0) break;
      const int g0 = s_g0[s];
      const bool active = tid < ng;
      int64_t row = 0;
      int g = 0, nk = 0;
      float4 f[5];
      if (active) {
        const uint32_t q = uint32_t(g0) + uint32_t(tid);
        const uint32_t dr = div_gpr(q);
        g = int(q - dr * uint32_t(gpr));
        row = s_row0[s] + dr;
        nk = int(min(int64_t(20), K - 20 * int64_t(g)));         // 4 .. 20, % 4 == 0
        const float4* src = reinterpret_cast<const float4*>(
            stage_smem + size_t(s) * kFuStageBytes + size_t(int(dr) * int(K) + 20 * (g - g0)) * 4);
#pragma unroll
        for (int v = 0; v < 5; ++v) f[v] = (4 * v < nk) ? src[v] : make_float4(0.f, 0.f, 0.f, 0.f);
      } else {
#pragma unroll
        for (int v = 0; v < 5; ++v) f[v] = make_float4(0.f, 0.f, 0.f, 0.f);
      }

      float y[4] = {0.f, 0.f, 0.f, 0.f};   // packed: per byte, sum of trit * 3^k
      float t8[20];                        // int8: the trits
      float nband = 0.f;                   // weights with T_lo <= |w| < T_hi
      float dot[kMM];                      // forward: sum_k t_k x_q[k]
#pragma unroll
      for (int m = 0; m < kMM; ++m) dot[m] = 0.f;
#pragma unroll
      for (int v = 0; v < 5; ++v) {
        float4 xv[kMM];
        if constexpr (kM > 0) {
#pragma unroll
          for (int m = 0; m < kM; ++m)
            xv[m] = active && 4 * v < nk ? reinterpret_cast<const float4*>(xf + int64_t(m) * K + 20 * g)[v]
                                         : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int P = 4 * v + j;
          const float x = f4get(f[v], j);
          const float ax = fabsf(x);
          if (P & 1)
            da1 = __dadd_rn(da1, double(ax));
          else
            da0 = __dadd_rn(da0, double(ax));
          const float mh = step_ge(ax, sc_hi);
          const float ml = step_ge(ax, sc_lo);
          nband = __fadd_rn(nband, __fsub_rn(ml, mh));
          const uint32_t sgn = __float_as_uint(x) & 0x80000000u;
          if (kPacked) {
            const float p3 = __uint_as_float(
                __float_as_uint(float(P % 5 == 0 ? 1 : P % 5 == 1 ? 3 : P % 5 == 2 ? 9 : P % 5 == 3 ? 27 : 81)) | sgn);
            y[P / 5] = __fmaf_rn(mh, p3, y[P / 5]);
          } else {
            t8[P] = __uint_as_float(__float_as_uint(mh) | sgn);
          }
          if constexpr (kM > 0) {
            const float t = __uint_as_float(__float_as_uint(mh) | sgn);
#pragma unroll
            for (int m = 0; m < kM; ++m) dot[m] = __fmaf_rn(t, f4get(xv[m], j), dot[m]);
          }
        }
      }
      if constexpr (kM > 0) {
#pragma unroll
        for (int m = 0; m < kM; ++m)
          add_by_row(a.yacc, int64_t(m) * N, active ? int(row) : -1, active ? __float2int_rn(dot[m]) : 0, lane);
      }
      // groups holding a band weight: one ballot, one list store per such lane
      const uint32_t pend = __ballot_sync(0xffffffffu, active && nband > 0.f);
      if (pend) {
        if (active && nband > 0.f) {
          const int pos = wcount + __popc(pend & ((1u << lane) - 1u));
          if (pos < cap_w) wl[pos] = (static_cast<unsigned long long>(row) << 32) | uint32_t(g);
        }
        wcount += __popc(pend);
      }
      if (active) {
        if (kPacked) {
          // byte = 121 + y: exact in the low mantissa bits of y + 2^23 + 121
          uint32_t vb[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) vb[j] = __float_as_uint(__fadd_rn(y[j], 8388729.0f));
          uint32_t* orow = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + row * ldo);
          orow[g] = __byte_perm(__byte_perm(vb[0], vb[1], 0x0040), __byte_perm(vb[2], vb[3], 0x0040), 0x5410);
          if (g == int(gpr) - 1)
            for (int64_t j = gpr; j < (ldo >> 2); ++j) orow[j] = 0x79797979u;  // pad bytes: 121
        } else {
          // int8 code = low byte of trit + 2^23 + 256
          uint32_t* o = reinterpret_cast<uint32_t*>(static_cast<int8_t*>(out) + row * ldo + 20 * g);
#pragma unroll
          for (int j = 0; j < 5; ++j) {
            uint32_t c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) c[i] = __float_as_uint(__fadd_rn(t8[4 * j + i], 8388864.0f));
            if (4 * j < nk)
              o[j] = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040), 0x5410);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // this warp is done with stage s
    }
    if (lane == 0 && wcount > cap_w) atomicOr(&acc->overflow, 1u);
  }
  __syncthreads();
  if (s_timeout && tid == 0) {
    // a wait gave up: report it, let every copy in flight land (bounded), and
    // still take part in the ticket, barrier B and the exit count so that the
    // workspace ends clear; mode 1 then re-codes everything
    raise_status(kDevTimeout);
    atomicOr(&acc->overflow, 2u);
    for (int s = 0; s < kStages; ++s)
      if (s_issued[s] > 0) (void)mbar_wait(&full[s], uint32_t(s_issued[s] - 1) & 1u);
  }

  // ---- end of phase 1: float64 CTA sum, ticket, the last CTA certifies beta ----
  {
    double d = __dadd_rn(da0, da1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) d = __dadd_rn(d, __shfl_down_sync(0xffffffffu, d, o));
    if (lane == 0) s_dpart[warp] = d;
  }
  __syncthreads();
  if (tid == 0) {
    double d = 0.0;
    for (int w = 0; w < kAbsThreads / 32; ++w) d = __dadd_rn(d, s_dpart[w]);
    atomicAdd(&acc->dsum, d);
    __threadfence();
    const unsigned int ticket = atomicAdd(&acc->ticket, 1u);   // grid barrier B: arrive
    if (ticket >= gridDim.x) raise_status(kDevBadWorkspace);
  }
  __threadfence();
  __syncthreads();
  // while the other CTAs finish: each lane loads its first listed group into
  // registers, and warms L2 with the rest of the list
  int64_t prow = -1, pg = 0;
  float4 pf[5];
  if (warp < kFuWarps) {
    const int cnt = min(wcount, cap_w);
    if (lane < cnt) {
      const unsigned long long ent = __ldcg(wl + lane);
      prow = int64_t(ent >> 32);
      pg = int64_t(ent & 0xFFFFFFFFull);
      const int nk = int(min(int64_t(20), K - 20 * pg));
      const float4* src = reinterpret_cast<const float4*>(W + prow * K + 20 * pg);
#pragma unroll
      for (int v = 0; v < 5; ++v) pf[v] = (4 * v < nk) ? ld_stream_f4(src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    for (int e = lane + 32; e < cnt; e += 32) {
      const unsigned long long ent = __ldcg(wl + e);
      const float* p = W + int64_t(ent >> 32) * K + 20 * int64_t(ent & 0xFFFFFFFFull);
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p + 19));
    }
  }
  if (tid == 0) {
    // barrier B: every CTA, once all have added their sums, certifies beta
    // itself from the same total (identical results everywhere)
    if (wait_u32_geq(&acc->ticket, gridDim.x)) {
      const double T = __ldcg(&acc->dsum);
      const unsigned int ovf = __ldcg(&acc->overflow);
      if (blockIdx.x == 0 && __ldcg(&acc->magic) != 0u) raise_status(kDevBadWorkspace);
      // longest addition chain: 10 per group in each of a thread's two sums (a
      // thread adds one group per chunk of its CTA: at most the static ones and
      // the whole tail), their sum, the warp tree, the warps, and one per CTA
      // at the atomic
      const double max_chunks = double(n_static) + double(nch - int64_t(n_static) * gridDim.x);
      const double L = 10.0 * max_chunks + 1.0 + 5.0 + double(kAbsThreads / 32) + double(gridDim.x);
      const double E = (L + 4.0) * 2.220446049250313e-16 * T;
      const float beta = certified_beta(T, E, n, eps);
      if (beta == beta) {
        if (blockIdx.x == 0) *beta_out = beta;
        s_beta = beta;
        const uint32_t tb = __float_as_uint(ternary_threshold(beta));
        const TernBand bd = s_band;
        s_mode = (bd.ok && bd.lo <= tb && tb <= bd.hi && ovf == 0u) ? 0 : 1;
        if (blockIdx.x == 0) acc->mode = uint32_t(s_mode);   // for inspection only
        s_next = 1;
      } else {
        s_next = 2;                          // not certified: everyone adds exactly
      }
    } else {
      raise_status(kDevTimeout);
      s_next = 0;                            // leave the provisional codes
    }
  }
  __syncthreads();

  // ---- (rare) exact pass: the absmean_kernel integer sum, grid-stride ----
  if (s_next == 2) {
    unsigned long long lo = 0ull;
    uint32_t hi = 0u;
    bool bad = false;
    const int64_t n4 = n >> 2;                        // n % 4 == 0, W 16-byte aligned
    for (int64_t i = int64_t(blockIdx.x) * blockDim.x + tid; i < n4; i += int64_t(gridDim.x) * blockDim.x) {
      const float4 v = ld_stream_f4(reinterpret_cast<const float4*>(W) + i);
      absmean_one(v.x, lo, hi, s_bins, bad);
      absmean_one(v.y, lo, hi, s_bins, bad);
      absmean_one(v.z, lo, hi, s_bins, bad);
      absmean_one(v.w, lo, hi, s_bins, bad);
    }
    const unsigned long long l0 = warp_sum_u64(lo & 0xFFFFFFFFull);
    const unsigned long long l1 = warp_sum_u64(lo >> 32);
    const unsigned long long l2 = warp_sum_u64((unsigned long long)hi);
    if (lane == 0) {
      s_wsum[3 * warp + 0] = l0;
      s_wsum[3 * warp + 1] = l1;
      s_wsum[3 * warp + 2] = l2;
    }
    if (__syncthreads_or(bad) && tid == 0) raise_status(kDevNonFinite);
    int any_bin = 0;
    for (int i = tid; i < 256; i += blockDim.x)
      if (s_bins[i]) {
        atomicAdd(&acc->bins[i], s_bins[i]);
        any_bin = 1;
      }
    if (any_bin) atomicOr(&acc->bins_used, 1u);
    if (tid < 3) {
      unsigned long long v = 0ull;
      for (int w = 0; w < kAbsThreads / 32; ++w) v += s_wsum[3 * w + tid];
      atomicAdd(&acc->tot[tid], v);
    }
    __threadfence();
    __syncthreads();
    if (tid == 0) s_last = atomicAdd(&acc->ticket2, 1u) == gridDim.x - 1;
    __syncthreads();
    if (s_last) {
      __threadfence();
      float beta;
      if (__ldcg(&acc->bins_used) != 0u) {
        // magnitudes outside the window: the general 512-bit rounding over the
        // limb totals (placed in slot 0) and the bins
        if (tid < 3) acc->slot[0][tid] = __ldcg(&acc->tot[tid]);
        __syncthreads();
        beta = absmean_finalize(acc, n, eps, beta_out, 1, s_binv, s_limb, s_wsum, s_word, s_big, &s_flag);
      } else {
        beta = tid == 0 ? beta_from_limbs(__ldcg(&acc->tot[0]), __ldcg(&acc->tot[1]), __ldcg(&acc->tot[2]),
                                          n, eps)
                        : 0.f;
        if (tid == 0) *beta_out = beta;
      }
      if (tid == 0) {
        s_beta = beta;
        const uint32_t tb = __float_as_uint(ternary_threshold(beta));
        const TernBand bd = s_band;
        s_mode = (bd.ok && bd.lo <= tb && tb <= bd.hi && __ldcg(&acc->overflow) == 0u) ? 0 : 1;
        acc->mode = uint32_t(s_mode);
        st_release_u32(&acc->flag_c, 1u);
        acc->tot[0] = 0ull;
        acc->tot[1] = 0ull;
        acc->tot[2] = 0ull;
        acc->bins_used = 0u;
        acc->ticket2 = 0u;
      }
    } else if (tid == 0) {
      if (wait_u32_geq(&acc->flag_c, 1u)) {
        s_mode = int(__ldcg(&acc->mode));
        s_beta = __ldcg(beta_out);
      } else {
        raise_status(kDevTimeout);
        s_next = 0;
      }
    }
    __syncthreads();
  }

  // ---- phase 2: re-code against the exact T (and correct the forward sums) ----
  if (s_next != 0) {
    const int mode = s_mode;
    const float T = ternary_threshold(s_beta);
    const StepConst sc_old = s_band.ok ? step_const(s_band.hi) : StepConst{__int_as_float(0x7F800000), 1.f};
    // one group: final codes into `out`; for the forward, the difference
    // between final and provisional codes dotted with the X codes
    auto recode = [&](int64_t row, int64_t g, const float4 (&w4)[5]) {
      const int nk = int(min(int64_t(20), K - 20 * g));
      if (kPacked) {
        uint32_t d[20];
#pragma unroll
        for (int P = 0; P < 20; ++P) d[P] = P < nk ? trit_digit(f4get(w4[P >> 2], P & 3), T) : 1u;
        uint32_t word = 0u;
#pragma unroll
        for (int b = 0; b < 4; ++b)
          word |= pack5_digits(d[5 * b], d[5 * b + 1], d[5 * b + 2], d[5 * b + 3], d[5 * b + 4]) << (8 * b);
        reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(out) + row * ldo)[g] = word;
      } else {
        uint32_t* o = reinterpret_cast<uint32_t*>(static_cast<int8_t*>(out) + row * ldo + 20 * g);
#pragma unroll
        for (int j = 0; j < 5; ++j)
          if (4 * j < nk)
            o[j] = uint32_t(uint8_t(trit_code(w4[j].x, T))) | uint32_t(uint8_t(trit_code(w4[j].y, T))) << 8 |
                   uint32_t(uint8_t(trit_code(w4[j].z, T))) << 16 | uint32_t(uint8_t(trit_code(w4[j].w, T))) << 24;
      }
      if constexpr (kM > 0) {
#pragma unroll
        for (int m = 0; m < kM; ++m) {
          float dd = 0.f;
#pragma unroll
          for (int P = 0; P < 20; ++P) {
            if (P < nk) {
              const float x = f4get(w4[P >> 2], P & 3);
              const float tdiff = float(trit_code(x, T)) - signed_step(x, sc_old);
              dd = __fmaf_rn(tdiff, xf[int64_t(m) * K + 20 * g + P], dd);
            }
          }
          const int di = __float2int_rn(dd);
          if (di != 0) atomicAdd(a.yacc + int64_t(m) * N + row, di);
        }
      }
    };
    if (mode == 0) {
      if (warp < kFuWarps) {
        const int cnt = min(wcount, cap_w);
        int e0 = lane;
        if (prow >= 0) {   // the preloaded group
          recode(prow, pg, pf);
          e0 = lane + 32;
        }
        for (int e = e0; e < cnt; e += 32) {
          const unsigned long long ent = __ldcg(wl + e);
          const int64_t row = int64_t(ent >> 32);
          const int64_t g = int64_t(ent & 0xFFFFFFFFull);
          const int nk = int(min(int64_t(20), K - 20 * g));
          const float4* src = reinterpret_cast<const float4*>(W + row * K + 20 * g);
          float4 w4[5];
#pragma unroll
          for (int v = 0; v < 5; ++v) w4[v] = (4 * v < nk) ? ld_stream_f4(src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
          recode(row, g, w4);
        }
      }
    } else if (kM == 0) {
      const int64_t t0 = int64_t(blockIdx.x) * blockDim.x + tid;
      const int64_t nthr = int64_t(gridDim.x) * blockDim.x;
      if (kPacked)
        ternarize_pack5_range(W, N, K, T, static_cast<uint8_t*>(out), ldo, t0, nthr);
      else
        ternarize_i8_range(W, n, T, static_cast<int8_t*>(out), t0, nthr);
    } else {
      // every group, with its forward correction; the pad words keep 121
      for (int64_t i = int64_t(blockIdx.x) * blockDim.x + tid; i < ngroups; i += int64_t(gridDim.x) * blockDim.x) {
        const int64_t row = i / gpr, g = i - row * gpr;
        const int nk = int(min(int64_t(20), K - 20 * g));
        const float4* src = reinterpret_cast<const float4*>(W + row * K + 20 * g);
        float4 w4[5];
#pragma unroll
        for (int v = 0; v < 5; ++v) w4[v] = (4 * v < nk) ? ld_stream_f4(src + v) : make_float4(0.f, 0.f, 0.f, 0.f);
        recode(row, g, w4);
      }
    }
  }
  // exit.  Plain quantizer: the CTA that leaves last clears the counters and
  // flags.  Forward: grid barrier C (every CTA's corrections are in), each CTA
  // writes its slice of Y = float(acc) (s beta) [+ b], and the CTA that finishes
  // that last clears the counters and flags.
  __threadfence();
  __syncthreads();
  unsigned int* const done = kM > 0 ? &acc->exit2 : &acc->exit_cnt;
  if constexpr (kM > 0) {
    if (tid == 0) {
      atomicAdd(&acc->exit_cnt, 1u);
      if (!wait_u32_geq(&acc->exit_cnt, gridDim.x)) raise_status(kDevTimeout);
    }
    __syncthreads();
    const float beta = s_beta;
    const int64_t per = ceil_div(N, int64_t(gridDim.x));
    const int64_t n0 = int64_t(blockIdx.x) * per, n1 = min(N, n0 + per);
#pragma unroll
    for (int m = 0; m < kM; ++m) {
      const float sb = __fmul_rn(s_xs[m], beta);
      for (int64_t i = n0 + tid; i < n1; i += blockDim.x) {
        float yv = __fmul_rn(float(__ldcg(a.yacc + int64_t(m) * N + i)), sb);
        if (a.bias) yv = __fadd_rn(yv, __ldg(a.bias + i));
        a.Y[int64_t(m) * N + i] = yv;
      }
    }
    __syncthreads();
  }
  if (tid == 0 && atomicAdd(done, 1u) == gridDim.x - 1) {
    acc->bar_a = 0u;
    acc->flag_c = 0u;
    acc->overflow = 0u;
    acc->exit_cnt = 0u;
    acc->exit2 = 0u;
    acc->ticket = 0u;
    acc->next_chunk = 0u;
    acc->dsum = 0.0;
  }
}

}  // namespace bl
