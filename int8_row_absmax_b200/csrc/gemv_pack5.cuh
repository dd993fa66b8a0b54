// Decode GEMV on packed trits: Y[m,:] = (x_q W_q^T)(s beta) [+ b] for M <= 4 rows.
//
// The deployed-path equation of "ultragraph -- when the graph is the 1-bit LLM,
// part 2" (section "autograd on a byte-graph") in the batch-1 decode regime the
// pages measure ("a 1-bit llm, from scratch": matvecs are most of the forward
// pass).  With M this small the layer streams the packed weights once, so the
// kernel is built around HBM bytes and the cost of decoding five trits per byte.
//
// Per CTA (one per SM, persistent over a contiguous block of rows):
//   * the rows' packed bytes arrive by 1-D bulk copies (TMA engine) into a ring
//     of shared-memory stages, all issued up front when they fit;
//   * the same kind of copy brings the float32 X rows into shared memory while
//     the CTA builds the decode table there; the CTA then quantizes X itself
//     (per-row absmax, then exactly the codes of bl_quantize_act) into a layout
//     matched to the decode;
//   * decode: a packed byte b holds digits d_k = floor(b/3^k) mod 3, trit t_k =
//     d_k - 1.  A 243-entry table gives (t0,t1,t2,t3) as four int8; every lane has
//     its own copy at b*256 + 4*lane, so 32 lanes never collide on a bank, and one
//     byte_perm forms the address.  The fifth digit d4 = floor(b/81) is computed
//     for four bytes at once: b*203 in 16-bit lanes puts d4 in bits 14..15
//     (exact for b <= 242), a byte_perm gathers those bytes and a mask keeps
//     64*d4.  Then sum_k t_k x_k = dp4a(table, x0..x3) + (dp4a(64 d4, x4) >> 6) - x4,
//     the last term summed once per row.
//   * each lane keeps the quantized x of its fixed 16-byte weight chunks in
//     registers and reuses them for every row; rows are reduced across the warp
//     with redux.sync and combined across K slices in shared memory.
#pragma once

#include "act_quant.cuh"
#include "common.cuh"
#include "ptx.cuh"

namespace bl {

constexpr int kGemvMaxM = 4;
constexpr int kGemvMaxWarps = 16;
constexpr int kLutBytes = 243 * 256;
constexpr int kGemvMaxSmem = 232448 - 1024;  // 227 KB per CTA, less the static arrays
constexpr int kGemvMaxRS = 32;

// The decode table as it sits in shared memory: word b*64 + l (l < 32) holds
// trits t0..t3 of byte b as int8, one copy per lane; words 32..63 of a row are
// unused, so the row pitch is 256 bytes and a byte_perm builds the address.
constexpr uint32_t kGemvXSmemMax = 64 * 1024;   // float32 X staged in shared memory up to this

struct GemvArgs {
  const float* X;       // [M,K] float32 (fused quantization) or nullptr
  const int8_t* Xq;     // [M,ldxq] int8 (pre-quantized) or nullptr
  int64_t ldxq;
  const uint8_t* Wp;    // [N,ldp]
  int64_t N, K, ldp;
  const float* beta;
  const float* bias;
  float eps;
  float* Y;             // [M,N] when dequantizing
  int32_t* acc;         // [M,N] when returning the integer product
  int S, slice, G, RS, nstage, rows_per_cta;
  uint32_t xstage_off, part_off, bar_off, stage_off, xf_off, xf_bytes;
};

struct GemvPlan {
  int M, CH, S, slice, G, nwarps, RS, nstage, rows_per_cta, grid;
  uint32_t xstage_off, part_off, bar_off, stage_off, xf_off, xf_bytes, smem;
};

inline uint32_t align_to(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Launch geometry for (M, N, K, ldp) on `sms` SMs; false if the GEMV cannot take it.
inline bool gemv_make_plan(int64_t M, int64_t N, int64_t K, int64_t ldp, int sms, GemvPlan& P,
                           bool x_copyable = false) {
  if (M < 1 || M > kGemvMaxM || N < 1 || K < 1 || ldp % 16 != 0) return false;
  const int64_t nch = ldp / 16;
  const int chmax = int(4 / M);                    // 20 * CH * M <= 80 x registers
  const int64_t S = ceil_div(nch, int64_t(32) * chmax);
  if (S > kGemvMaxWarps) return false;
  P.M = int(M);
  P.S = int(S);
  P.slice = int(ceil_div(nch, S));
  P.CH = int(ceil_div(P.slice, 32));
  P.G = S >= 16 ? 1 : int(16 / S);
  P.nwarps = P.S * P.G;
  const int64_t grid0 = N < sms ? N : sms;
  P.rows_per_cta = int(ceil_div(N, grid0));
  P.grid = int(ceil_div(N, P.rows_per_cta));
  int64_t rs = 16384 / ldp;
  rs = rs < 1 ? 1 : (rs > kGemvMaxRS ? kGemvMaxRS : rs);
  if (rs > P.rows_per_cta) rs = P.rows_per_cta;
  P.RS = int(rs);
  P.xf_bytes = (x_copyable && M * K * 4 <= kGemvXSmemMax) ? uint32_t(M * K * 4) : 0u;
  P.xf_off = align_to(kLutBytes, 128);
  P.xstage_off = align_to(P.xf_off + P.xf_bytes, 128);
  P.part_off = align_to(P.xstage_off + uint32_t(M * 5 * ldp), 16);
  P.bar_off = align_to(P.part_off + uint32_t(M * P.RS * 4), 16);
  const int64_t nst = ceil_div(P.rows_per_cta, P.RS);
  const uint32_t stage_bytes = uint32_t(P.RS * ldp);
  int64_t ns = nst < 8 ? nst : 8;
  for (; ns >= 1; --ns) {
    P.stage_off = align_to(P.bar_off + uint32_t(8 * (ns + 1)), 128);
    if (int64_t(P.stage_off) + ns * stage_bytes <= kGemvMaxSmem) break;
  }
  if (ns < 1) return false;
  P.nstage = int(ns);
  P.smem = uint32_t(P.stage_off + ns * stage_bytes);
  return true;
}

// Whether some launch geometry fits (independent of the SM count).
inline bool gemv_feasible(int64_t M, int64_t N, int64_t K, int64_t ldp) {
  GemvPlan P;
  return gemv_make_plan(M, 1, K, ldp, 1, P) && N >= 1;
}

__device__ __forceinline__ uint32_t byte_perm(uint32_t a, uint32_t b, uint32_t s) {
  return __byte_perm(a, b, s);
}

template <int M, int CH, bool kFused, bool kDequant>
__global__ void __launch_bounds__(kGemvMaxWarps * 32, 1) gemv_pack5_kernel(const GemvArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ float s_redf[M * kGemvMaxWarps];
  __shared__ int s_redi[M * kGemvMaxWarps];
  __shared__ float s_scale[M];
  __shared__ int s_x4sum[M];

  uint32_t* xst = reinterpret_cast<uint32_t*>(smem + a.xstage_off);
  int* part = reinterpret_cast<int*>(smem + a.part_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + a.bar_off);
  unsigned char* stages = smem + a.stage_off;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nthr = blockDim.x;
  const int64_t ldp = a.ldp, K = a.K;
  const int64_t row0 = int64_t(blockIdx.x) * a.rows_per_cta;
  const int rows = int(min(int64_t(a.rows_per_cta), a.N - row0));
  const int RS = a.RS, nstage = a.nstage;
  const int nst = (rows + RS - 1) / RS;
  const uint32_t stage_bytes = uint32_t(RS * ldp);

  auto issue = [&](int st, int buf) {
    const int r = st * RS;
    const int nr = min(RS, rows - r);
    const uint32_t bytes = uint32_t(nr * ldp);
    mbar_arrive_expect_tx(&bars[buf], bytes);
    bulk_g2s(stages + size_t(buf) * stage_bytes, a.Wp + (row0 + r) * ldp, bytes, &bars[buf]);
  };

  // 1. barriers, then the table / X copy and every weight copy that fits
  uint64_t* bar_x = &bars[nstage];
  if (tid == 0) {
    for (int s = 0; s <= nstage; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0) {
    if (a.xf_bytes) {
      mbar_arrive_expect_tx(bar_x, a.xf_bytes);
      bulk_g2s(smem + a.xf_off, a.X, a.xf_bytes, bar_x);
    }
    for (int s = 0; s < nstage && s < nst; ++s) issue(s, s);
  }
  for (int i = tid; i < M * RS; i += nthr) part[i] = 0;
  // the decode table, built in place while the copies fly: word b*64 + l holds
  // trits t0..t3 of byte b (one copy per lane l).  Lane l of a warp computes the
  // word of byte 32 i + l once; shuffles spread each word to its 32 slots.
  for (int blk = warp; blk < 8; blk += nthr >> 5) {
    const uint32_t bl = uint32_t(blk * 32 + lane);
    const uint32_t b1 = (bl * 171u) >> 9, b2 = (bl * 57u) >> 9, b3 = (bl * 19u) >> 9;  // bl/3, /9, /27
    const uint32_t d0 = bl - 3u * b1, d1 = b1 - 3u * b2, d2 = b2 - 3u * b3, d3 = b3 - 3u * ((bl * 203u) >> 14);
    const uint32_t v = ((d0 + 255u) & 0xFFu) | ((d1 + 255u) & 0xFFu) << 8 | ((d2 + 255u) & 0xFFu) << 16 |
                       ((d3 + 255u) & 0xFFu) << 24;
#pragma unroll 8
    for (int i = 0; i < 32; ++i) {
      const uint32_t e = uint32_t(blk * 32 + i);
      const uint32_t vi = __shfl_sync(0xffffffffu, v, i);
      if (e < 243u) reinterpret_cast<uint32_t*>(smem)[e * 64u + uint32_t(lane)] = vi;
    }
  }
  const bool xready = a.xf_bytes ? mbar_wait(bar_x, 0u) : true;
  if (!__syncthreads_and(xready)) {
    if (tid == 0) {
      raise_status(kDevTimeout);
      for (int s2 = 0; s2 < nst && s2 < nstage; ++s2) (void)mbar_wait(&bars[s2], 0u);
    }
    return;
  }

  // 2. quantized x in decode order: for weight word g (packed bytes 4g..4g+3,
  //    weights 20g..20g+19) five words: x[5j..5j+3] for j = 4g+i (i<4), then
  //    x[5j+4] for the four j.  Element k = 5j + r goes to byte 20g + 4i + r
  //    (r < 4) or 20g + 16 + i (r = 4); positions past K hold 0.  Four elements
  //    per thread and step, all rows.
  const int kpad = int(5 * ldp);
  unsigned char* xb = reinterpret_cast<unsigned char*>(xst);
  const float* xsrc = a.xf_bytes ? reinterpret_cast<const float*>(smem + a.xf_off) : a.X;
  float scm[M];
  if (kFused) {
    const bool xvec = aligned(xsrc, 16) && (K & 3) == 0;
    const int64_t K4 = xvec ? (K >> 2) : 0;
    float amax[M];
    bool bad = false;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      amax[m] = 0.f;
      const float* xr = xsrc + int64_t(m) * K;
      for (int64_t i = tid; i < K4; i += nthr) {
        const float4 v = reinterpret_cast<const float4*>(xr)[i];
        const float mx = fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
        bad |= !(mx <= 3.402823466e38f) | (v.x != v.x) | (v.y != v.y) | (v.z != v.z) | (v.w != v.w);
        amax[m] = fmaxf(amax[m], mx);
      }
      for (int64_t i = (K4 << 2) + tid; i < K; i += nthr) {
        const float v = fabsf(xr[i]);
        bad |= !(v <= 3.402823466e38f);
        amax[m] = fmaxf(amax[m], v);
      }
      const float w = warp_max(amax[m]);
      if (lane == 0) s_redf[m * kGemvMaxWarps + warp] = w;
    }
    if (__syncthreads_or(bad) && tid == 0) raise_status(kDevNonFinite);
    // every warp forms the row scales from the per-warp maxima (no extra barrier)
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float w = warp_max(lane < (nthr >> 5) ? s_redf[m * kGemvMaxWarps + lane] : 0.f);
      scm[m] = __fadd_rn(__fdiv_rn(w, float(kActQmax)), a.eps);
      if (tid == 0) s_scale[m] = scm[m];
    }
  }
  int x4part[M];
#pragma unroll
  for (int m = 0; m < M; ++m) {
    x4part[m] = 0;
    unsigned char* xbm = xb + int64_t(m) * kpad;
    const float* xr = kFused ? xsrc + int64_t(m) * K : nullptr;
    const int8_t* xq = kFused ? nullptr : a.Xq + int64_t(m) * a.ldxq;
    const float sc = kFused ? scm[m] : 0.f, rc = kFused ? act_recip(sc) : 0.f;
    for (int i4 = tid; i4 < (kpad >> 2); i4 += nthr) {
      const int k = 4 * i4;
      uint32_t c[4];
      if (kFused) {
        bool tie = rc == 0.f;
        if (k + 4 <= K && aligned(xr + k, 16)) {
          const float4 f = *reinterpret_cast<const float4*>(xr + k);
          c[0] = act_code_try(f.x, rc, tie);
          c[1] = act_code_try(f.y, rc, tie);
          c[2] = act_code_try(f.z, rc, tie);
          c[3] = act_code_try(f.w, rc, tie);
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) c[e] = k + e < K ? act_code_try(xr[k + e], rc, tie) : 0u;
        }
        if (tie)   // rare: a quotient near a half-integer; exact division
          for (int e = 0; e < 4 && k + e < K; ++e) c[e] = uint32_t(uint8_t(int8_t(act_code_slow(xr[k + e], sc))));
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) c[e] = k + e < K ? uint32_t(uint8_t(xq[k + e])) : 0u;
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t kk = uint32_t(k + e);
        const uint32_t j = __umulhi(kk, 0xCCCCCCCDu) >> 2;     // kk / 5
        const uint32_t r = kk - 5u * j;
        const uint32_t off = 20u * (j >> 2) + (r < 4u ? 4u * (j & 3u) + r : 16u + (j & 3u));
        xbm[off] = uint8_t(c[e]);
        if (r == 4u) x4part[m] += int(int8_t(uint8_t(c[e])));
      }
    }
  }
#pragma unroll
  for (int m = 0; m < M; ++m) {
    int v = x4part[m];
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) s_redi[m * kGemvMaxWarps + warp] = v;
  }
  __syncthreads();
  if (tid < M) {
    int t = 0;
    for (int w = 0; w < nthr / 32; ++w) t += s_redi[tid * kGemvMaxWarps + w];
    s_x4sum[tid] = t;
  }

  // 4. this lane's x registers: chunks c0 + lane + 32 i of its K slice
  const int sl = warp % a.S, grp = warp / a.S;
  const int64_t nch = ldp / 16;
  const int64_t c0 = int64_t(sl) * a.slice;
  const int64_t c1 = min(nch, c0 + a.slice);
  uint32_t xr[M][CH][20];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const int64_t c = c0 + lane + 32 * i;
      const uint4* src = reinterpret_cast<const uint4*>(xb + int64_t(m) * kpad + 80 * c);
#pragma unroll
      for (int v = 0; v < 5; ++v) {
        const uint4 u = (c < c1) ? src[v] : make_uint4(0u, 0u, 0u, 0u);
        xr[m][i][4 * v + 0] = u.x;
        xr[m][i][4 * v + 1] = u.y;
        xr[m][i][4 * v + 2] = u.z;
        xr[m][i][4 * v + 3] = u.w;
      }
    }
  const uint32_t lanebase = uint32_t(lane) * 4u;
  const float beta = kDequant ? *a.beta : 0.f;

  // 5. stream the stages
#pragma unroll 1
  for (int st = 0; st < nst; ++st) {
    const int buf = st % nstage;
    const uint32_t parity = uint32_t(st / nstage) & 1u;
    const bool ok = mbar_wait(&bars[buf], parity);
    if (!__syncthreads_and(ok)) {
      if (tid == 0) {
        raise_status(kDevTimeout);
        for (int s2 = st + 1; s2 < nst && s2 < st + nstage; ++s2)
          (void)mbar_wait(&bars[s2 % nstage], uint32_t(s2 / nstage) & 1u);
      }
      return;
    }
    const unsigned char* sbuf = stages + size_t(buf) * stage_bytes;
    const int nr = min(RS, rows - st * RS);
#pragma unroll 1
    for (int rl = grp; rl < nr; rl += a.G) {
      const unsigned char* rowp = sbuf + int64_t(rl) * ldp;
      int am[M], a4[M];
#pragma unroll
      for (int m = 0; m < M; ++m) am[m] = a4[m] = 0;
#pragma unroll
      for (int i = 0; i < CH; ++i) {
        const int64_t c = c0 + lane + 32 * i;
        if (c < c1) {
          const uint4 w4 = *reinterpret_cast<const uint4*>(rowp + 16 * c);
          const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const uint32_t w = wv[q];
            uint32_t t[4];
#pragma unroll
            for (int bb = 0; bb < 4; ++bb)
              t[bb] = *reinterpret_cast<const uint32_t*>(smem + byte_perm(w, lanebase, 0x5504u | (bb << 4)));
            const uint32_t E = byte_perm(w, 0u, 0x4240u) * 203u;
            const uint32_t O = byte_perm(w, 0u, 0x4341u) * 203u;
            const uint32_t D = byte_perm(E, O, 0x7351u) & 0xC0C0C0C0u;
#pragma unroll
            for (int m = 0; m < M; ++m) {
              int acc = am[m];
#pragma unroll
              for (int bb = 0; bb < 4; ++bb) acc = __dp4a(int(t[bb]), int(xr[m][i][5 * q + bb]), acc);
              am[m] = acc;
              a4[m] = dp4a_us(D, xr[m][i][5 * q + 4], a4[m]);
            }
          }
        }
      }
#pragma unroll
      for (int m = 0; m < M; ++m) {
        const int tot = __reduce_add_sync(0xffffffffu, am[m] + (a4[m] >> 6));
        if (lane == 0) atomicAdd(&part[m * RS + rl], tot);
      }
    }
    __syncthreads();
    for (int t = tid; t < nr * M; t += nthr) {
      const int m = t / nr, rl = t - m * nr;
      const int acc = part[m * RS + rl] - s_x4sum[m];
      part[m * RS + rl] = 0;
      const int64_t n = row0 + int64_t(st) * RS + rl;
      if (kDequant) {
        float y = __fmul_rn(float(acc), __fmul_rn(s_scale[m], beta));
        if (a.bias) y = __fadd_rn(y, a.bias[n]);
        a.Y[m * a.N + n] = y;
      } else {
        a.acc[m * a.N + n] = acc;
      }
    }
    __syncthreads();
    if (tid == 0 && st + nstage < nst) {
      fence_proxy_async_smem();
      issue(st + nstage, buf);
    }
  }
}

}  // namespace bl
