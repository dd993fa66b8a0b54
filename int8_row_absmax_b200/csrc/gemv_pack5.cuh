// Decode GEMV on packed trits: Y[m,:] = (x_q W_q^T)(s beta) [+ b] for M <= 4 rows.
//
// The deployed-path equation of "ultragraph -- when the graph is the 1-bit LLM,
// part 2" (section "autograd on a byte-graph") in the batch-1 decode regime the
// pages measure ("a 1-bit llm, from scratch": matvecs are most of the forward
// pass).  With M this small the layer streams the packed weights once, so the
// kernel is built around HBM bytes and the cost of decoding five trits per byte.
//
// One launch serves up to kGemvMaxProbs independent problems (each CTA belongs
// to one problem and owns a contiguous block of its rows), so several layers
// that read different activations (for instance the projections that share
// one input) stream their weights in one grid.
//
// Per CTA (one per SM):
//   * before the dependency wait (programmatic dependent launch): mbarriers;
//   * griddepcontrol.wait, then launch_dependents (the next kernel may start
//     its own prologue while this one computes); thread 0 issues the copy of X
//     first (X is on the critical path, and every copy issued ahead of it --
//     weights included, even with static weights -- was measured to delay it),
//     then the segments of packed rows (bulk copies into shared memory) and,
//     last, a bulk copy of the decode table (a compile-time constant in global
//     memory), which is needed only once the activation codes are ready;
//   * X: per-row absmax over the whole row (every CTA reads it, from L2), then
//     exactly the codes of bl_quantize_act, stored in shared memory in decode
//     order: for packed word g (bytes 4g..4g+3, trits 20g..20g+19) five words,
//     x[5j..5j+3] for j = 4g+i (i < 4), then x[5j+4] of the four j;
//   * decode: a packed byte b holds digits d_k = floor(b/3^k) mod 3, trit
//     t_k = d_k - 1.  A 243-entry table gives (t0,t1,t2,t3) as four int8; every
//     lane has its own copy at b*256 + 4*lane, so the 32 lanes never collide on
//     a bank and one byte_perm forms the address.  The fifth digit d4 =
//     floor(b/81) comes four bytes at a time: b*203 in 16-bit lanes holds it in
//     bits 14..15 (exact for b <= 242), a byte_perm gathers those bytes and a
//     mask keeps 64*d4.  So sum_k t_k x_k = dp4a(table, x0..x3) +
//     (dp4a(64 d4, x4) >> 6) - x4, the last term summed once per row;
//   * each lane keeps the codes of its fixed 16-byte weight chunks in registers
//     for every row; S warps share a row (one K slice each), G rows are in flight
//     per CTA, partial sums meet in shared memory; Y is written at the end.
#pragma once

#include "act_quant.cuh"
#include "common.cuh"
#include "ptx.cuh"
#include "trit_table.cuh"

namespace bl {

constexpr int kGemvMaxM = 4;
constexpr int kGemvWarps = 16;
constexpr int kGemvThreads = kGemvWarps * 32;
constexpr int kGemvMaxProbs = 4;
constexpr uint32_t kGemvMaxSmem = 232448 - 1024;  // 227 KB per CTA, less the static arrays
constexpr uint32_t kGemvSegTarget = 128 * 1024;  // bytes per bulk copy (one mbarrier each): few, large copies
constexpr uint32_t kGemvSegMin = 4 * 1024;
constexpr int kGemvMaxStages = 24;
constexpr uint32_t kGemvXStageMax = 64 * 1024;  // float32 X rows staged in shared memory up to this

struct GemvProb {
  const float* X;      // [M, K] float32 (activation quantization inside) or nullptr
  const int8_t* Xq;    // [M, ldxq] int8 codes (given) or nullptr
  int64_t ldxq;
  const uint8_t* Wp;   // [N, ldp] packed trits
  int64_t N, K, ldp;
  const float* beta;
  const float* bias;
  float* Y;            // [M, N] float32 output, or nullptr
  int32_t* acc;        // [M, N] int32 integer product when Y is nullptr
  float eps;
  int cta0;            // first CTA of this problem
  int rows_per_cta;
  int S, G;            // warps per row slice, rows in flight
  int slice;           // 16-byte chunks per row slice: ceil(ldp / 16 / S)
  int seg_rows, nstage;
  uint32_t xc_off, xs_off, xs_bytes, part_off, bar_off, stage_off, smem;
};

struct GemvArgs {
  GemvProb p[kGemvMaxProbs];
  int nprob;
};

inline uint32_t align_to(uint32_t v, uint32_t a) { return (v + a - 1) / a * a; }

// Chunks of 16 packed bytes per lane, for M rows and a row of ldp bytes: the
// fewest that let at most 16 warps cover a row (every warp keeps the codes of
// its own chunks in registers, and all of them are read from shared memory
// once per warp), up to 4 / M (20 code words per chunk and row, at most 80).
inline int gemv_chunks_per_lane(int64_t M, int64_t ldp) {
  const int64_t nch = ldp / 16;
  for (int64_t ch = 1; ch <= 4 / M; ++ch)
    if (ceil_div(nch, int64_t(32) * ch) <= kGemvWarps) return int(ch);
  return 0;
}

// Rows a warp works on at once (independent chains of loads and dp4a): three
// for one row of X and one chunk per lane (measured: 6.30 us for the decode step
// against 6.34 with two and 6.77 with four).
__host__ __device__ constexpr int gemv_rows_per_pass(int M, int CH) { return M * CH == 1 ? 3 : (M * CH >= 4 ? 1 : 4 / (M * CH)); }

// The weights' segment ring of a problem whose other offsets are set: rows per
// warp group and segment are at least one pass of gemv_rows_per_pass rows.
// Fewer, larger copies were measured faster (each costs its issuing thread
// time), so the largest segment target that either holds all of the CTA's rows
// at once or still gives a ring of three stages; failing both, the smallest
// target that fits at all.  False if no ring fits.
inline bool gemv_plan_ring(int64_t M, int64_t ldp, int ch, GemvProb& P) {
  P.part_off = align_to(P.xs_off + P.xs_bytes, 16);
  P.bar_off = align_to(P.part_off + uint32_t(M * P.rows_per_cta * 4), 16);
  const int64_t rpp = gemv_rows_per_pass(int(M), ch);
  bool found = false;
  for (uint32_t target = kGemvSegTarget; target >= kGemvSegMin; target /= 2) {
    int64_t per = int64_t(target) / (int64_t(P.G) * ldp);
    per = per < rpp ? rpp : per / rpp * rpp;
    int64_t seg = P.G * per;
    if (seg > P.rows_per_cta) seg = P.rows_per_cta;
    const int64_t nseg = ceil_div(P.rows_per_cta, seg);
    const uint32_t stage_bytes = uint32_t(seg * ldp);
    int64_t ns = nseg < kGemvMaxStages ? nseg : kGemvMaxStages;
    uint32_t stage_off = 0;
    for (; ns >= 1; --ns) {
      stage_off = align_to(P.bar_off + uint32_t(8 * (ns + 2)), 128);
      if (int64_t(stage_off) + ns * stage_bytes <= kGemvMaxSmem) break;
    }
    if (ns < 1) continue;
    P.stage_off = stage_off;
    P.seg_rows = int(seg);
    P.nstage = int(ns);
    P.smem = uint32_t(stage_off + ns * stage_bytes);
    found = true;
    if (ns >= nseg || ns >= 3) break;
  }
  return found;
}

// Geometry of one problem on `ctas` CTAs: warps per slice, row groups, the
// segment ring and the shared-memory layout.  False if the GEMV cannot take it.
inline bool gemv_plan_prob(int64_t M, int64_t N, int64_t K, int64_t ldp, int ctas, int ch,
                           GemvProb& P) {
  if (M < 1 || M > kGemvMaxM || N < 1 || K < 1 || ldp % 16 != 0 || ldp * 5 < K || ctas < 1) return false;
  const int64_t nch = ldp / 16;
  const int64_t S = ceil_div(nch, int64_t(32) * ch);
  if (S > kGemvWarps) return false;
  P.S = int(S);
  P.G = kGemvWarps / P.S;
  P.slice = int(ceil_div(nch, S));
  P.rows_per_cta = int(ceil_div(N, int64_t(ctas)));
  P.xc_off = align_to(kLutBytes, 128);
  P.xs_off = align_to(P.xc_off + uint32_t(M * 5 * ldp), 16);
  // X staged in shared memory when it fits (and the weights' ring still does),
  // else read from global memory
  const bool stage_x = uint64_t(M * K * 4) <= kGemvXStageMax && K % 4 == 0;
  for (int attempt = stage_x ? 0 : 1; attempt < 2; ++attempt) {
    P.xs_bytes = attempt == 0 ? uint32_t(M * K * 4) : 0u;
    if (gemv_plan_ring(M, ldp, ch, P)) return true;
  }
  return false;
}

// CTAs of one GEMV launch (split over its problems by the launch's time
// model).  Planned for B200's 148 SMs (a fixed figure, so that plans and
// the feasibility test need no device query; on a smaller device the extra
// CTAs simply queue, since GEMV CTAs never wait on one another).
constexpr int kGemvCtas = 148;

// Whether some launch geometry takes (M, N, K, ldp).
inline bool gemv_feasible(int64_t M, int64_t N, int64_t K, int64_t ldp) {
  const int ch = gemv_chunks_per_lane(M, ldp);
  GemvProb P;
  return ch > 0 && gemv_plan_prob(M, N, K, ldp, int(N < kGemvCtas ? N : kGemvCtas), ch, P);
}

template <int M, int CH, bool kFused, int kMinBlocks>
__global__ void __launch_bounds__(kGemvThreads, kMinBlocks) gemv_pack5_kernel(const __grid_constant__ GemvArgs a) {
  extern __shared__ __align__(1024) unsigned char smem[];
  __shared__ float s_red[M * kGemvWarps];
  __shared__ float s_scale[M];
  __shared__ int s_x4[M];
  __shared__ int s_fail;

  int pi = 0;
#pragma unroll
  for (int i = 1; i < kGemvMaxProbs; ++i)
    if (i < a.nprob && int(blockIdx.x) >= a.p[i].cta0) pi = i;
  const GemvProb& P = a.p[pi];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t ldp = P.ldp, K = P.K;
  const int rpc = P.rows_per_cta;
  const int64_t row0 = int64_t(int(blockIdx.x) - P.cta0) * rpc;
  const int rows = int(min(int64_t(rpc), P.N - row0));
  const int seg_rows = P.seg_rows, nstage = P.nstage;
  const int nseg = (rows + seg_rows - 1) / seg_rows;
  const bool ring = nseg > nstage;
  unsigned char* xc = smem + P.xc_off;
  int* part = reinterpret_cast<int*>(smem + P.part_off);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P.bar_off);
  unsigned char* stages = smem + P.stage_off;
  const uint32_t stage_bytes = uint32_t(seg_rows) * uint32_t(ldp);

  int issued = 0;                 // segments copied so far (thread 0)
  auto issue = [&](int sg) {
    ++issued;
    const int buf = sg % nstage;
    const int r = sg * seg_rows;
    const uint32_t bytes = uint32_t(min(seg_rows, rows - r)) * uint32_t(ldp);
    mbar_arrive_expect_tx(&bars[buf], bytes);
    bulk_g2s(stages + size_t(buf) * stage_bytes, P.Wp + (row0 + r) * ldp, bytes, &bars[buf]);
  };

  // ---- prologue: nothing here reads what an earlier kernel may still write
  uint64_t* bar_x = &bars[nstage];
  uint64_t* bar_lut = &bars[nstage + 1];
  if (tid == 0) {
    for (int s = 0; s <= nstage + 1; ++s) mbar_init(&bars[s], 1);
    fence_mbar_init();
    s_fail = 0;
  }
  if (tid < M) s_x4[tid] = 0;

  griddep_wait();                 // X and W may come from the previous kernel
  griddep_launch_dependents();
  // float32 X into shared memory by one bulk copy (one latency for the whole row)
  const bool staged = kFused && P.xs_bytes != 0u;
  if (tid == 0) {
    if (staged) {
      mbar_arrive_expect_tx(bar_x, P.xs_bytes);
      bulk_g2s(smem + P.xs_off, P.X, P.xs_bytes, bar_x);
    }
    for (int sg = 0; sg < nseg && sg < nstage; ++sg) issue(sg);
    // the decode table last: it is needed only once the codes are ready
    mbar_arrive_expect_tx(bar_lut, kLutBytes);
    bulk_g2s(smem, &g_trit_lut, kLutBytes, bar_lut);
  }
  for (int i = tid; i < M * rpc; i += kGemvThreads) part[i] = 0;
  __syncthreads();                // the mbarriers are initialized before any thread polls one
  if (!__syncthreads_and(staged ? mbar_wait(bar_x, 0u) : true)) {
    if (tid == 0) {
      raise_status(kDevTimeout);
      (void)mbar_wait(bar_lut, 0u);
      for (int sg = issued > nstage ? issued - nstage : 0; sg < issued; ++sg)
        (void)mbar_wait(&bars[sg % nstage], uint32_t(sg / nstage) & 1u);
    }
    return;
  }

  // ---- activations: codes in decode order, sum of the fifth-position codes
  const int kpad = int(5 * ldp);
  float scm[M];
  const float* xsrc = staged ? reinterpret_cast<const float*>(smem + P.xs_off) : P.X;
  // 16-byte loads of X through generic addresses, valid for the staged copy
  // in shared memory and for global memory alike (four per thread issued
  // together, so the latencies overlap); no global-only load form here
  auto ld4 = [](const float* p) -> float4 { return *reinterpret_cast<const float4*>(p); };
  if (kFused) {
    const bool xvec = aligned(P.X, 16) && (K & 3) == 0;
    const int64_t K4 = xvec ? (K >> 2) : 0;
    bool bad = false;
#pragma unroll
    for (int m = 0; m < M; ++m) {
      float amax = 0.f;
      const float* xr = xsrc + int64_t(m) * K;
      for (int64_t i0 = tid; i0 < K4; i0 += 4 * kGemvThreads) {
        float4 v[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t i = i0 + int64_t(u) * kGemvThreads;
          v[u] = i < K4 ? ld4(xr + 4 * i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const float mx = fmaxf(fmaxf(fabsf(v[u].x), fabsf(v[u].y)), fmaxf(fabsf(v[u].z), fabsf(v[u].w)));
          bad |= !(mx <= 3.402823466e38f) | (v[u].x != v[u].x) | (v[u].y != v[u].y) | (v[u].z != v[u].z) |
                 (v[u].w != v[u].w);
          amax = fmaxf(amax, mx);
        }
      }
      for (int64_t i = (K4 << 2) + tid; i < K; i += kGemvThreads) {
        const float v = fabsf(xr[i]);
        bad |= !(v <= 3.402823466e38f);
        amax = fmaxf(amax, v);
      }
      amax = warp_max(amax);
      if (lane == 0) s_red[m * kGemvWarps + warp] = amax;
    }
    if (__syncthreads_or(bad) && tid == 0) raise_status(kDevNonFinite);
#pragma unroll
    for (int m = 0; m < M; ++m) {
      const float w = warp_max(lane < kGemvWarps ? s_red[m * kGemvWarps + lane] : 0.f);
      scm[m] = __fadd_rn(__fdiv_rn(w, float(kActQmax)), P.eps);
      if (tid == 0) s_scale[m] = scm[m];
    }
  }
  // codes in decode order, one packed byte's five activations per thread (the
  // most threads the row allows): byte j = 4 g + i of packed word g puts its
  // first four codes in word i of the word's five (xc + 20 g + 4 i) and its
  // fifth code in byte i of the fifth word
  const int nbyte = int(ldp);
#pragma unroll
  for (int m = 0; m < M; ++m) {
    int x4 = 0;
    unsigned char* xcm = xc + m * kpad;
    const float* xr = kFused ? xsrc + int64_t(m) * K : nullptr;
    const int8_t* xq = kFused ? nullptr : P.Xq + int64_t(m) * P.ldxq;
    const float sc = kFused ? scm[m] : 0.f, rc = kFused ? act_recip(sc) : 0.f;
    for (int j = tid; j < nbyte; j += kGemvThreads) {
      const int k0 = 5 * j;
      uint32_t c[5];
      if (kFused) {
        float xv[5];
#pragma unroll
        for (int e = 0; e < 5; ++e) xv[e] = k0 + e < K ? xr[k0 + e] : 0.f;
        act_codes_n<5>(xv, int(min(int64_t(5), K - int64_t(k0))), sc, rc, c);
      } else {
#pragma unroll
        for (int e = 0; e < 5; ++e) c[e] = k0 + e < K ? uint32_t(uint8_t(xq[k0 + e])) : 0u;
      }
      unsigned char* dst = xcm + 20 * (j >> 2);
      *reinterpret_cast<uint32_t*>(dst + 4 * (j & 3)) = pack_code_bytes(c[0], c[1], c[2], c[3]);
      dst[16 + (j & 3)] = uint8_t(c[4]);
      x4 += int(int8_t(uint8_t(c[4])));
    }
    x4 = __reduce_add_sync(0xffffffffu, x4);
    if (lane == 0 && x4) atomicAdd(&s_x4[m], x4);
  }
  __syncthreads();

  // ---- this lane's x registers: chunks c0 + lane + 32 i of its K slice
  const int S = P.S, G = P.G;
  const int grp = warp / S, sl = warp - grp * S;
  const int nch = int(ldp >> 4);
  const int c0 = sl * P.slice;
  const int c1 = min(nch, c0 + P.slice);
  uint32_t xr[M][CH][20];
#pragma unroll
  for (int m = 0; m < M; ++m)
#pragma unroll
    for (int i = 0; i < CH; ++i) {
      const int c = c0 + lane + 32 * i;
      const uint4* src = reinterpret_cast<const uint4*>(xc + m * kpad + 80 * c);
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

  // ---- stream the segments (the table first; ok is CTA-uniform: the ring's
  // loop has barriers)
  bool ok = __syncthreads_and(mbar_wait(bar_lut, 0u));
#pragma unroll 1
  for (int sg = 0; sg < nseg && ok; ++sg) {
    const int buf = sg % nstage;
    if (!mbar_wait(&bars[buf], uint32_t(sg / nstage) & 1u)) {
      ok = false;
      if (!ring) break;
    }
    if (ring && !__syncthreads_and(ok)) break;
    const unsigned char* sbuf = stages + size_t(buf) * stage_bytes;
    const int r0 = sg * seg_rows;
    const int nr = min(seg_rows, rows - r0);
    if (grp < G) {
      // kRows rows per pass (rl, rl + G, ...) and two accumulators per row and x
      // row (even and odd words): independent chains of table loads and dp4a
      constexpr int kRows = gemv_rows_per_pass(M, CH);
#pragma unroll 1
      for (int rl = grp; rl < nr; rl += kRows * G) {
        const unsigned char* rowp[kRows];
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr)
          rowp[rr] = sbuf + int64_t(rl + rr * G < nr ? rl + rr * G : rl) * ldp;
        int am[kRows][M][2], a4[kRows][M];
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr)
#pragma unroll
          for (int m = 0; m < M; ++m) am[rr][m][0] = am[rr][m][1] = a4[rr][m] = 0;
#pragma unroll
        for (int i = 0; i < CH; ++i) {
          const int c = c0 + lane + 32 * i;
          if (c < c1) {
            uint32_t wv[kRows][4];
#pragma unroll
            for (int rr = 0; rr < kRows; ++rr) {
              const uint4 w4 = *reinterpret_cast<const uint4*>(rowp[rr] + 16 * c);
              wv[rr][0] = w4.x;
              wv[rr][1] = w4.y;
              wv[rr][2] = w4.z;
              wv[rr][3] = w4.w;
            }
#pragma unroll
            for (int q = 0; q < 4; ++q) {
#pragma unroll
              for (int rr = 0; rr < kRows; ++rr) {
                const uint32_t w = wv[rr][q];
                uint32_t t[4];
#pragma unroll
                for (int bb = 0; bb < 4; ++bb) t[bb] = lut_t0123(smem, w, lanebase, bb);
                const uint32_t D = d4x64(w);
#pragma unroll
                for (int m = 0; m < M; ++m) {
                  int acc = am[rr][m][q & 1];
#pragma unroll
                  for (int bb = 0; bb < 4; ++bb) acc = __dp4a(int(t[bb]), int(xr[m][i][5 * q + bb]), acc);
                  am[rr][m][q & 1] = acc;
                  a4[rr][m] = dp4a_us(D, xr[m][i][5 * q + 4], a4[rr][m]);
                }
              }
            }
          }
        }
#pragma unroll
        for (int rr = 0; rr < kRows; ++rr) {
          const int row_l = rl + rr * G;
#pragma unroll
          for (int m = 0; m < M; ++m) {
            const int tot = __reduce_add_sync(0xffffffffu, am[rr][m][0] + am[rr][m][1] + (a4[rr][m] >> 6));
            if (lane == 0 && row_l < nr) {
              if (S == 1) part[m * rpc + r0 + row_l] = tot;
              else atomicAdd(&part[m * rpc + r0 + row_l], tot);
            }
          }
        }
      }
    }
    if (ring) {
      __syncthreads();              // every warp is done with this buffer
      if (tid == 0 && sg + nstage < nseg) {
        fence_proxy_async_smem();
        issue(sg + nstage);
      }
    }
  }
  if (!ok) s_fail = 1;
  __syncthreads();
  if (s_fail) {
    // a copy never landed: let the ones still in flight finish, write nothing
    if (tid == 0) {
      raise_status(kDevTimeout);
      (void)mbar_wait(bar_lut, 0u);
      for (int sg = issued > nstage ? issued - nstage : 0; sg < issued; ++sg)
        (void)mbar_wait(&bars[sg % nstage], uint32_t(sg / nstage) & 1u);
    }
    return;
  }

  // ---- epilogue: y = float32(acc) (s beta) [+ b], or the integer product
  const float beta = kFused ? *P.beta : 0.f;
  for (int t = tid; t < rows * M; t += kGemvThreads) {
    const int m = t / rows, rl = t - m * rows;
    const int acc = part[m * rpc + rl] - s_x4[m];
    const int64_t n = row0 + rl;
    if (kFused) {
      float y = __fmul_rn(float(acc), __fmul_rn(s_scale[m], beta));
      if (P.bias) y = __fadd_rn(y, P.bias[n]);
      P.Y[m * P.N + n] = y;
    } else {
      P.acc[m * P.N + n] = acc;
    }
  }
}

}  // namespace bl
