// Single-launch prepass: K channel mean, Q/K INT8 and V E4M3 quantisation in
// one cooperative kernel in which every byte of Q, K and V is read from HBM
// once.
//
// Operation: the same steps and rounding as the separate prepass kernels
// ("Sage2 Blackwell Mainloop", sections "Decision" and "Existing
// Contract"), fused into one producer as the pages' P1/P2 producer fusions
// do ("Sage2 Blackwell Mainloop", section "Completed P1 And P2").  Bytes and
// scales equal those of the separate kernels.
//
// Layout of the work.  A cooperative launch of G CTAs, two per SM, all
// resident together.  CTA i owns a fixed run of 64-token chunks,
// [i*T64/G, (i+1)*T64/G), in every head; its slice of one head's K or V is
// at most 32 KB.  Heads (units u = b*H + h) are taken g at a time
// ("groups") in two passes, K with Q, then V.  The two warpgroups of a CTA
// form a two-stage pipeline over the steps (one group each):
//   - warps 0-7 (statistics): wait for the slices of step s, compute their
//     statistics (K: FP64 chunk sums, V: absolute maxima), publish them with
//     atomics and count the CTA in; then wait (bounded) until all G CTAs
//     have counted in for step s-1 and form its K means or V scales;
//   - warps 8-15 (quant): copy the slices of step s+1 into one of three
//     shared-memory slots (cp.async), quantise the Q rows of step s (K
//     pass), then quantise K or V of step s-1 from the slices that are still
//     resident.
// So K and V are read once, and the statistics of one group overlap the
// quantisation of the previous one.

// The K mean.  The definition is the FP64 sum of the FP64 chunk partials
// in chunk order, each partial a token-order FP64 sum, divided by N in FP64
// and rounded once to FP32.  The chunk partials are computed exactly so.  A
// nonzero partial p is a multiple of 2^lo(p), its lowest set bit, and below
// 2^(hi(p)+1) in magnitude; with lo and hi the minimum and maximum over a
// channel's chunks, every sum of partials is a multiple of 2^lo below
// 2^(ceil(log2 T64)+hi+1), so it is exact in FP64 when
// ceil(log2 T64) + hi - lo <= 52.  Then any order of adding the partials
// gives the chunk-order sum, bit for bit.  Each CTA therefore adds its
// partials (in order) into an FP64 accumulator with an atomic add and
// publishes hi and lo with atomic maxima; a channel within the bound takes
// its mean from the accumulator.  For a channel outside it, the CTAs add
// the partials (written to k_part) in chunk order, one warp per channel.
// Every CTA computes the same means; CTA 0 stores them.
//
// Waits.  A CTA only waits for counts that every CTA reaches without
// waiting on anything itself: the statistics of step s come before its wait
// at step s.  Each wait is bounded (the status word records
// SAGE_ERR_TIMEOUT, a global abort flag stops the others, and every CTA
// leaves after draining its own copies).
#include <algorithm>

#include "prepass_codes.cuh"
#include "tc_prims.cuh"

namespace sage {
namespace {

constexpr int kRThreads = 512;
constexpr int kCtasPerSm = 2;
constexpr int kSlotBytes = 32 * 1024;
constexpr int kSlots = 3;
constexpr int kMaxSliceChunkD = kSlotBytes / (kKTile * 2);  // max chunks x D of one slice (256)

struct ResArgs {
  const uint16_t *q, *k, *v;
  int64_t qsb, qsn, qsh, ksb, ksn, ksh, vsb, vsn, vsh;
  int N, H, U, Nq, Nk, T64, TQ, G32;
  int G;      // CTAs
  int g;      // units per group
  int S;      // groups per pass
  int cpc;    // most K/V chunks of one CTA
  int cpcq;   // most Q chunks of one CTA
  int log2t;  // ceil(log2 T64)
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  float* k_mean;
  uint8_t* v8;
  float* v_scale;
  double* k_part;  // [U][T64][D] FP64 chunk partials (read only for channels off the bound)
  double* k_sum;   // [U][D] zeroed
  int* k_hi;       // [U][D] zeroed: kExpBias + max over chunks of floor(log2 |partial|)
  int* k_lov;      // [U][D] zeroed: kExpBias - min over chunks of the lowest set bit (0: all partials 0)
  int* v_amax;     // [U][D] zeroed: FP32 bits of the channel amax
  int* arrive;     // [2][U] zeroed: CTAs counted in (K, V)
  int* abort_flag; // [1] zeroed
  DeviceStatus* status;
  long long wait_limit;
  int stall_unit;  // test hook: CTA 0 does not count in for the K of this unit (-1: none)
};

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// Shared-memory image of a slice: token rows of D BF16 values; the 16-byte
// piece k of row r is stored at position k ^ ((r >> 4) & 3), so that reads
// down a channel (16 tokens per lane, four 16-token runs per warp) and reads
// along a row both fall in distinct banks.
template <int D>
__device__ __forceinline__ uint32_t slice_off(int r, int piece) {
  return (uint32_t)(r * D * 2 + ((piece ^ ((r >> 4) & 3)) << 4));
}

struct Range {
  int lo, n;  // first chunk and chunk count of this CTA
};
__device__ __forceinline__ Range cta_range(int total, int G) {
  const int i = blockIdx.x;
  const int lo = (int)((long long)i * total / G), hi = (int)((long long)(i + 1) * total / G);
  return {lo, hi - lo};
}

// Copies of the K (kind 0) or V (kind 1) slices of group grp into a slot,
// issued by the Q warps only: the statistics warps, whose thread 0 releases
// the CTA's counts, then have no copies in flight for that release to wait
// on.
template <int D>
__device__ void issue_slices(const ResArgs& a, int kind, int grp, uint8_t* slot, Range r) {
  constexpr int SEG = D / 8;
  const uint16_t* base = kind == 0 ? a.k : a.v;
  const int64_t sb = kind == 0 ? a.ksb : a.vsb, sn = kind == 0 ? a.ksn : a.vsn, sh = kind == 0 ? a.ksh : a.vsh;
  if (threadIdx.x < kRThreads / 2) return;  // statistics warps
  const int per_unit = r.n * kKTile * SEG;
  const uint32_t s0 = smem_u32(slot);
  for (int i = 0; i < a.g; ++i) {
    const int u = grp * a.g + i;
    if (u >= a.U) break;
    const uint16_t* ub = base + (u / a.H) * sb + (u % a.H) * sh;
    const uint32_t sd = s0 + (uint32_t)(i * a.cpc * kKTile * D * 2);
    for (int idx = threadIdx.x - kRThreads / 2; idx < per_unit; idx += kRThreads / 2) {
      const int row = idx / SEG, piece = idx % SEG;
      const int n = r.lo * kKTile + row;
      const bool valid = n < a.N;
      cp_async_16_zfill(sd + slice_off<D>(row, piece), valid ? ub + (int64_t)n * sn + piece * 8 : base, valid);
    }
  }
}

// Warps 0-7 ("statistics warps") and warps 8-15 ("Q warps") synchronise
// among themselves with named barriers while the other half works.
constexpr int kHalf = kRThreads / 2;
constexpr int kBarStats = 1, kBarQ = 2;
__device__ __forceinline__ void bar_half(int id) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(kHalf) : "memory"); }

__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));  // a NaN operand yields the other
  return d;
}

// Bounded wait (thread 0) until all CTAs have counted in for every unit of a
// group; the statistics warps then pass a named barrier.  Returns false (in
// every statistics thread) when the wait ran out or another CTA gave up.
__device__ bool wait_group(const ResArgs& a, int kind, int grp, int* s_flag) {
  if (threadIdx.x == 0) {
    int good = 1;
    for (int i = 0; i < a.g && good; ++i) {
      const int u = grp * a.g + i;
      if (u >= a.U) break;
      const int* cnt = a.arrive + kind * a.U + u;
      const long long t0 = clock64();
      for (unsigned it = 0;; ++it) {
        int c;
        asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(c) : "l"(cnt) : "memory");
        if (c >= a.G) break;
        if (*reinterpret_cast<volatile int*>(a.abort_flag)) {
          good = 0;
          break;
        }
        if (clock64() - t0 > a.wait_limit) {
          good = 0;
          if (atomicCAS(&a.status->code, 0, (int)SAGE_ERR_TIMEOUT) == 0) {
            a.status->where = 40 + kind;
            a.status->block = (int)blockIdx.x;
          }
          atomicExch(a.abort_flag, 1);
          break;
        }
        __nanosleep(it < 8 ? 32 : 256);
      }
    }
    *s_flag = good;
  }
  bar_half(kBarStats);
  return *s_flag != 0;
}

// Count this CTA in for each unit of the group.  Called by the statistics
// warps after a named barrier that follows all their writes and atomics:
// thread 0's release is cumulative over what the barrier ordered before it.
__device__ void count_in(const ResArgs& a, int kind, int grp) {
  if (threadIdx.x == 0) {
    for (int i = 0; i < a.g; ++i) {
      const int u = grp * a.g + i;
      if (u >= a.U) break;
      if (kind == 0 && u == a.stall_unit && blockIdx.x == 0) continue;
      int* cnt = a.arrive + kind * a.U + u;
      asm volatile("red.release.gpu.global.add.s32 [%0], 1;" ::"l"(cnt) : "memory");
    }
  }
}

// ------------------------------------------------------------ statistics
// Statistics thread t < 256 takes channels d, d+1 (d even) of one chunk of
// one unit: the two FP64 token-order sums (K) or absolute maxima (V).
// Rows come 16 at a time, whose pieces share one swizzle.
//
// K also reports, per channel, floor(log2 |p|) and the exponent of the
// lowest set bit of each nonzero chunk partial p (atomic maxima of kExpBias
// + hi and kExpBias - lo), which the K mean's exactness test needs.

template <int D>
__device__ __noinline__ void k_stats(const ResArgs& a, int grp, const uint8_t* slot, Range r, double* sp) {
  const int t = threadIdx.x;
  const int item = t / (D / 2), d = 2 * (t % (D / 2));
  const int i = item / a.cpc, cc = item % a.cpc;
  const int u = grp * a.g + i;
  double p0 = 0.0, p1 = 0.0;
  if (i < a.g && u < a.U && cc < r.n) {
    const uint8_t* s = slot + i * a.cpc * kKTile * D * 2 + ((d & 7) << 1);
#pragma unroll
    for (int r0 = cc * kKTile; r0 < cc * kKTile + kKTile; r0 += 16) {
      const uint8_t* rp = s + slice_off<D>(r0, d >> 3);
#pragma unroll
      for (int j = 0; j < 16; ++j) {  // token order; pad rows hold zeros
        const uint32_t w = *reinterpret_cast<const uint32_t*>(rp + j * D * 2);
        p0 = __dadd_rn(p0, (double)__uint_as_float(w << 16));
        p1 = __dadd_rn(p1, (double)__uint_as_float(w & 0xFFFF0000u));
      }
    }
    *reinterpret_cast<double2*>(a.k_part + ((size_t)u * a.T64 + r.lo + cc) * D + d) = make_double2(p0, p1);
  }
  if (item < a.g * a.cpc) {
    sp[item * D + d] = p0;
    sp[item * D + d + 1] = p1;
  }
  bar_half(kBarStats);
  if (t < a.g * D / 2) {
    const int i2 = t / (D / 2), d2 = 2 * (t % (D / 2)), u2 = grp * a.g + i2;
    if (u2 < a.U) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        double sum = 0.0;
        int hi = 0, lov = 0;
        for (int c = 0; c < r.n; ++c) {  // the CTA's chunks in order
          const double p = sp[(i2 * a.cpc + c) * D + d2 + h];
          sum = __dadd_rn(sum, p);
          if (p != 0.0) {
            int ph, pl;
            partial_bits(p, ph, pl);
            hi = max(hi, kExpBias + ph);
            lov = max(lov, kExpBias - pl);
          }
        }
        const size_t at = (size_t)u2 * D + d2 + h;
        atomicAdd(a.k_sum + at, sum);
        if (lov) {
          atomicMax(a.k_hi + at, hi);
          atomicMax(a.k_lov + at, lov);
        }
      }
    }
  }
  bar_half(kBarStats);
}

template <int D>
__device__ __noinline__ void v_stats(const ResArgs& a, int grp, const uint8_t* slot, Range r, float* sf) {
  const int t = threadIdx.x;
  const int item = t / (D / 2), d = 2 * (t % (D / 2));
  const int i = item / a.cpc, cc = item % a.cpc;
  const int u = grp * a.g + i;
  uint32_t m = 0u;
  if (i < a.g && u < a.U && cc < r.n) {
    const uint8_t* s = slot + i * a.cpc * kKTile * D * 2 + ((d & 7) << 1);
#pragma unroll
    for (int r0 = cc * kKTile; r0 < cc * kKTile + kKTile; r0 += 16) {
      const uint8_t* rp = s + slice_off<D>(r0, d >> 3);
#pragma unroll
      for (int j = 0; j < 16; ++j)
        m = max_bf16x2(m, *reinterpret_cast<const uint32_t*>(rp + j * D * 2) & 0x7FFF7FFFu);
    }
  }
  if (item < a.g * a.cpc) {
    sf[item * D + d] = __uint_as_float(m << 16);
    sf[item * D + d + 1] = __uint_as_float(m & 0xFFFF0000u);
  }
  bar_half(kBarStats);
  if (t < a.g * D / 2) {
    const int i2 = t / (D / 2), d2 = 2 * (t % (D / 2)), u2 = grp * a.g + i2;
    if (u2 < a.U) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float mxv = 0.0f;
        for (int c = 0; c < r.n; ++c) mxv = fmaxf(mxv, sf[(i2 * a.cpc + c) * D + d2 + h]);
        // the amax of non-negative floats is exact in any order, and their
        // bit patterns order as integers
        if (mxv > 0.0f) atomicMax(a.v_amax + (size_t)u2 * D + d2 + h, __float_as_int(mxv));
      }
    }
  }
  bar_half(kBarStats);
}

// ---------------------------------------------------------------------- Q
// The Q warps (256 threads): D threads per 64-row chunk, 8 pieces of 16
// bytes each (pieces tt + D * j: rows tt/(D/8) + 8j, so j < 4 lie in the
// first 32-row group and j >= 4 in the second).  The loads are issued at the
// start of the step and used after the K slice has arrived.
constexpr int kQPieces = 8;

template <int D>
__device__ void q_load(const ResArgs& a, int grp, Range rq, uint4 (&x)[kQPieces]) {
  constexpr int SEG = D / 8, TPI = D;
  const int qt = threadIdx.x - kHalf;
  const int item = qt / TPI, tt = qt % TPI, col = (tt % SEG) * 8;
  const int i = item / a.cpcq, cc = item % a.cpcq;
  const int u = grp * a.g + i;
  const bool live = i < a.g && u < a.U && cc < rq.n;
  const int b = live ? u / a.H : 0, h = live ? u % a.H : 0;
#pragma unroll
  for (int j = 0; j < kQPieces; ++j) {
    const int row = (rq.lo + cc) * kKTile + tt / SEG + 8 * j;
    x[j] = live && row < a.N ? ldg16(a.q + b * a.qsb + (int64_t)row * a.qsn + h * a.qsh + col)
                             : make_uint4(0, 0, 0, 0);
  }
}

template <int D>
__device__ void q_quant(const ResArgs& a, int grp, Range rq, const uint4 (&x)[kQPieces], uint32_t* redq,
                        int* s_any) {
  constexpr int SEG = D / 8, TPI = D, WPI = TPI / 32, HALF = kQPieces / 2;
  const int qt = threadIdx.x - kHalf, qw = qt >> 5, lane = qt & 31;
  const int item = qt / TPI, tt = qt % TPI, col = (tt % SEG) * 8;
  const int i = item / a.cpcq, cc = item % a.cpcq;
  const int u = grp * a.g + i;
  const bool live = i < a.g && u < a.U && cc < rq.n;
  // amax as BF16 magnitude bits (NaN and inf above every finite value)
  uint32_t mb[2] = {0u, 0u};
#pragma unroll
  for (int j = 0; j < kQPieces; ++j) mb[j / HALF] = amax_bits8(x[j], mb[j / HALF]);
  mb[0] = __reduce_max_sync(0xffffffffu, halves_max(mb[0]));
  mb[1] = __reduce_max_sync(0xffffffffu, halves_max(mb[1]));
  if (qt == 0) *s_any = 0;
  if (lane == 0) {
    redq[2 * qw] = mb[0];
    redq[2 * qw + 1] = mb[1];
  }
  bar_half(kBarQ);
  float am[2];
  bool finite[2];
#pragma unroll
  for (int gg = 0; gg < 2; ++gg) {
    uint32_t m = redq[2 * (item * WPI) + gg];
#pragma unroll
    for (int w = 1; w < WPI; ++w) m = max(m, redq[2 * (item * WPI + w) + gg]);
    finite[gg] = m < 0x7F80u;
    am[gg] = __uint_as_float(m << 16);
    if (!finite[gg]) *s_any = 1;
  }
  bar_half(kBarQ);
  if (*s_any) {
    // NaN or inf among the rows: the amax that ignores NaN (the reference form)
    float af[2] = {0.0f, 0.0f};
#pragma unroll
    for (int j = 0; j < kQPieces; ++j) {
      float f[8];
      unpack_bf16x8(x[j], f);
#pragma unroll
      for (int e = 0; e < 8; ++e) af[j / HALF] = fmaxf(af[j / HALF], fabsf(f[e]));
    }
    af[0] = warp_max(af[0]);
    af[1] = warp_max(af[1]);
    float* redf = reinterpret_cast<float*>(redq) + 16;
    if (lane == 0) {
      redf[2 * qw] = af[0];
      redf[2 * qw + 1] = af[1];
    }
    bar_half(kBarQ);
#pragma unroll
    for (int gg = 0; gg < 2; ++gg) {
      float m = redf[2 * (item * WPI) + gg];
#pragma unroll
      for (int w = 1; w < WPI; ++w) m = fmaxf(m, redf[2 * (item * WPI + w) + gg]);
      am[gg] = m;
    }
  }
  float inv[2];
  bool fast[2];
#pragma unroll
  for (int gg = 0; gg < 2; ++gg) {
    inv[gg] = am[gg] > 0.0f ? __fdiv_rn(127.0f, am[gg]) : 0.0f;
    fast[gg] = finite[gg] && codes_fast(am[gg], inv[gg]);
    const int grp32 = 2 * (rq.lo + cc) + gg;
    if (live && tt == 0 && grp32 < a.G32)
      a.q_scale[(size_t)u * a.G32 + grp32] = am[gg] > 0.0f ? __fdiv_rn(am[gg], 127.0f) : 0.0f;
  }
  if (live) {
    int8_t* dst = a.q8 + ((size_t)u * a.Nq + (size_t)(rq.lo + cc) * kKTile) * D + col;
#pragma unroll
    for (int j = 0; j < kQPieces; ++j) {
      const int rr = tt / SEG + 8 * j;
      float f[8];
      unpack_bf16x8(x[j], f);  // pad rows were loaded as zeros: zero codes
      *reinterpret_cast<uint2*>(dst + (size_t)rr * D) =
          fast[j / HALF] ? i8_codes8_fast(f, inv[j / HALF]) : i8_codes8_ref(f, inv[j / HALF]);
    }
  }
}

// ------------------------------------------------------------------ K mean
// Statistics warps: the mean of every channel of the group's units into
// mean_s[i * D + d] (all CTAs compute the same values; CTA 0 stores them).
template <int D>
__device__ __noinline__ void k_means(const ResArgs& a, int grp, float* mean_s, int* list, int* s_cnt) {
  const int t = threadIdx.x;
  if (t == 0) *s_cnt = 0;
  bar_half(kBarStats);
  for (int c = t; c < a.g * D; c += kHalf) {
    const int u = grp * a.g + c / D;
    if (u >= a.U) break;
    const size_t at = (size_t)u * D + c % D;
    const int hi = __ldcg(a.k_hi + at) - kExpBias, lov = __ldcg(a.k_lov + at);
    // every partial is a multiple of 2^lo and below 2^(hi+1) in magnitude, so
    // every sum of partials is a multiple of 2^lo below 2^(log2t + hi + 1):
    // exact in FP64 when log2t + hi - lo <= 52, and then the accumulator
    // holds the chunk-order sum (all partials zero: +0)
    if (lov == 0 || partials_exact(a.log2t, hi, kExpBias - lov)) {
      mean_s[c] = lov == 0 ? 0.0f : __double2float_rn(__ddiv_rn(__ldcg(a.k_sum + at), (double)a.N));
    } else {
      list[atomicAdd(s_cnt, 1)] = c;
    }
  }
  bar_half(kBarStats);
  const int nlist = *s_cnt;
  if (nlist > 0) {
    // channels off the bound: the chunk partials added in chunk order, one
    // warp per channel (lanes load 32 chunks at a time; every lane adds the
    // same values in the same order, so all hold the same total)
    const int warp = t >> 5, lane = t & 31;
    for (int e = warp; e < nlist; e += kHalf / 32) {
      const int c = list[e];
      const int u = grp * a.g + c / D, d = c % D;
      const double* src = a.k_part + (size_t)u * a.T64 * D + d;
      double total = 0.0;
      double nxt = lane < a.T64 ? __ldcg(src + (size_t)lane * D) : 0.0;
      for (int c0 = 0; c0 < a.T64; c0 += 32) {
        const double cur = nxt;
        if (c0 + 32 + lane < a.T64) nxt = __ldcg(src + (size_t)(c0 + 32 + lane) * D);
        const int n = min(32, a.T64 - c0);
        for (int j = 0; j < n; ++j) total = __dadd_rn(total, __shfl_sync(0xffffffffu, cur, j));
      }
      if (lane == 0) mean_s[c] = __double2float_rn(__ddiv_rn(total, (double)a.N));
    }
    bar_half(kBarStats);
  }
  if (blockIdx.x == 0)
    for (int c = t; c < a.g * D; c += kHalf) {
      const int u = grp * a.g + c / D;
      if (u < a.U) a.k_mean[(size_t)u * D + c % D] = mean_s[c];
    }
}

// Statistics warps: 448 / amax of every channel of the group's units into
// vinv_s (CTA 0 also stores the scales amax / 448).
template <int D>
__device__ void v_scales(const ResArgs& a, int grp, float* vinv_s) {
  for (int c = threadIdx.x; c < a.g * D; c += kHalf) {
    const int u = grp * a.g + c / D;
    if (u >= a.U) break;
    const float am = __int_as_float(__ldcg(a.v_amax + (size_t)u * D + c % D));
    vinv_s[c] = am > 0.0f ? __fdiv_rn(448.0f, am) : 0.0f;
    if (blockIdx.x == 0) a.v_scale[(size_t)u * D + c % D] = am > 0.0f ? __fdiv_rn(am, 448.0f) : 0.0f;
  }
}

// K (quant warps): 2D threads per 64-row chunk from the resident slice;
// x' = fl32(x - km).
template <int D>
__device__ void k_quant(const ResArgs& a, int grp, const uint8_t* slot, Range r, const float* kmean_s, float* red,
                        int* s_any) {
  constexpr int SEG = D / 8, TPI = 2 * D, WPI = TPI / 32, IPP = kHalf / TPI;
  constexpr int PER = kKTile * SEG / TPI;  // 4
  const int qt = threadIdx.x - kHalf;
  const int tt = qt % TPI, piece = tt % SEG, col = piece * 8;
  uint32_t* redb = reinterpret_cast<uint32_t*>(red);
  const int items = a.g * a.cpc;
  for (int it0 = 0; it0 < items; it0 += IPP) {
    const int item = it0 + qt / TPI;
    const int i = item / a.cpc, cc = item % a.cpc;
    const int u = grp * a.g + i;
    const bool live = item < items && u < a.U && cc < r.n;
    uint4 xr[PER];
    float km[8];
    float amax = 0.0f;  // NaN-propagating
    if (live) {
      const uint8_t* s = slot + i * a.cpc * kKTile * D * 2;
#pragma unroll
      for (int j = 0; j < 8; ++j) km[j] = kmean_s[i * D + col + j];
#pragma unroll
      for (int p = 0; p < PER; ++p) {
        const int rr = (tt + TPI * p) / SEG;
        xr[p] = *reinterpret_cast<const uint4*>(s + slice_off<D>(cc * kKTile + rr, piece));
        if ((r.lo + cc) * kKTile + rr < a.N) {
          float f[8];
          unpack_bf16x8(xr[p], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) amax = fmax_nan(amax, fabsf(__fsub_rn(f[j], km[j])));
        }
      }
    }
    // the bits of non-negative floats order as integers, NaN above inf
    const uint32_t ab = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
    if (qt == 0) *s_any = 0;
    if ((qt & 31) == 0) redb[qt >> 5] = ab;
    bar_half(kBarQ);
    const uint32_t* rb = redb + (qt / TPI) * WPI;
    uint32_t m = rb[0];
#pragma unroll
    for (int w = 1; w < WPI; ++w) m = max(m, rb[w]);
    const bool finite = m < 0x7F800000u;
    amax = __uint_as_float(m);
    if (!finite) *s_any = 1;
    bar_half(kBarQ);
    if (*s_any) {
      // NaN or inf among the rows: the amax that ignores NaN (the reference form)
      float af = 0.0f;
      if (live)
#pragma unroll
        for (int p = 0; p < PER; ++p) {
          const int rr = (tt + TPI * p) / SEG;
          if ((r.lo + cc) * kKTile + rr < a.N) {
            float f[8];
            unpack_bf16x8(xr[p], f);
#pragma unroll
            for (int j = 0; j < 8; ++j) af = fmaxf(af, fabsf(__fsub_rn(f[j], km[j])));
          }
        }
      af = warp_max(af);
      if ((qt & 31) == 0) red[16 + (qt >> 5)] = af;
      bar_half(kBarQ);
      const float* rw = red + 16 + (qt / TPI) * WPI;
      amax = rw[0];
#pragma unroll
      for (int w = 1; w < WPI; ++w) amax = fmaxf(amax, rw[w]);
    }
    bar_half(kBarQ);  // red is reused by the next items
    if (live) {
      const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
      const bool fast = finite && codes_fast(amax, inv);
      if (tt == 0) a.k_scale[(size_t)u * a.T64 + r.lo + cc] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
      int8_t* dst = a.k8 + ((size_t)u * a.Nk + (size_t)(r.lo + cc) * kKTile) * D;
#pragma unroll
      for (int p = 0; p < PER; ++p) {
        const int rr = (tt + TPI * p) / SEG;
        uint2 o = make_uint2(0u, 0u);  // pad rows get zero codes
        if ((r.lo + cc) * kKTile + rr < a.N) {
          float f[8], x[8];
          unpack_bf16x8(xr[p], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) x[j] = __fsub_rn(f[j], km[j]);
          o = fast ? i8_codes8_fast(x, inv) : i8_codes8_ref(x, inv);
        }
        *reinterpret_cast<uint2*>(dst + (size_t)rr * D + col) = o;
      }
    }
  }
}

// V (quant warps): runs of 16 tokens of one channel from the resident slice converted to
// E4M3 (token t in byte t of the channel's row) and stored as one 16-byte
// vector; a warp covers four runs of eight channels (64 contiguous bytes
// per channel).
template <int D>
__device__ void v_quant(const ResArgs& a, int grp, const uint8_t* slot, Range r, const float* vinv_s) {
  constexpr int SEG = D / 8;
  const int runs = a.g * a.cpc * 4 * D;
  for (int idx = threadIdx.x - kHalf; idx < runs; idx += kHalf) {
    const int q = idx & 3, cl = (idx >> 2) & 7, rest = idx >> 5;
    const int cb = rest % SEG, item = rest / SEG;
    const int i = item / a.cpc, cc = item % a.cpc;
    const int u = grp * a.g + i;
    if (u >= a.U || cc >= r.n) continue;
    const int ch = cb * 8 + cl;
    const float inv = vinv_s[i * D + ch];
    const uint8_t* s = slot + i * a.cpc * kKTile * D * 2;
    const int t0 = cc * kKTile + 16 * q;  // (t >> 4) & 3 == q for the run's tokens
    const uint16_t* colp = reinterpret_cast<const uint16_t*>(s + (((cb ^ q) << 4) + (cl << 1)));
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int tk = t0 + 4 * j;
      const uint32_t lo = e4m3x2(__fmul_rn(bf16_bits_to_f32(colp[tk * D]), inv),
                                 __fmul_rn(bf16_bits_to_f32(colp[(tk + 1) * D]), inv));
      const uint32_t hi = e4m3x2(__fmul_rn(bf16_bits_to_f32(colp[(tk + 2) * D]), inv),
                                 __fmul_rn(bf16_bits_to_f32(colp[(tk + 3) * D]), inv));
      w[j] = inv > 0.0f ? (lo | (hi << 16)) : 0u;
    }
    uint8_t* dst = a.v8 + ((size_t)u * D + ch) * a.Nk + (size_t)(r.lo + cc) * kKTile + 16 * q;
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// Dynamic shared memory: the slots, then the scratch.
constexpr size_t kScratchOff = (size_t)kSlots * kSlotBytes;
constexpr size_t kSmemBytes = kScratchOff + kMaxSliceChunkD * sizeof(double)  // sp (FP64 partials / FP32 maxima)
                              + 2 * kMaxSliceChunkD * sizeof(float)            // mean_buf[2] (K means / V 448/amax)
                              + kMaxSliceChunkD * sizeof(int)                  // list
                              + 64 * sizeof(float);                            // red (K: 32), redq (Q: 32)

// The two warpgroups run as a pipeline, handing over through mbarriers:
//   statistics warps, step st: wait for the slices of step st; statistics;
//     count in; wait (bounded) for all CTAs' counts of step st-1; its K
//     means or V inverse scales into mean_buf[(st-1) & 1]; means_ready.
//   quant warps, step st: copies of step st+1 into the slot that step st-2
//     left; in the K pass the Q rows of step st; wait for means_ready of
//     step st-1, quantise its slices; means_free.
// Slot st % 3 is written by the copies of step st, read by the statistics of
// step st and by the quantisation at quant step st+1, and refilled at quant
// step st+2, after this warpgroup's own quantisation of it.
struct Pipe {
  uint64_t slot_full[kSlots];  // the copies of a slot have landed (256 cp.async arrivals)
  uint64_t means_ready[2];     // mean_buf[b] holds the means of the next step to quantise
  uint64_t means_free[2];      // the quant warps are done with mean_buf[b]
  int abort;                   // CTA-local: a bounded wait gave up
  int flag;                    // 0 once the statistics warps' global wait failed
  int cnt, anyq, anyk;
};

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int D>
__global__ void __launch_bounds__(kRThreads, kCtasPerSm) prepass_resident_kernel(const __grid_constant__ ResArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  double* sp = reinterpret_cast<double*>(smem + kScratchOff);
  float* mean_buf = reinterpret_cast<float*>(sp + kMaxSliceChunkD);  // [2][kMaxSliceChunkD]
  int* list = reinterpret_cast<int*>(mean_buf + 2 * kMaxSliceChunkD);
  float* red = reinterpret_cast<float*>(list + kMaxSliceChunkD);
  uint32_t* redq = reinterpret_cast<uint32_t*>(red + 32);
  __shared__ Pipe pp;
  volatile int* abort_cta = &pp.abort;

  const Range rk = cta_range(a.T64, a.G);
  const Range rq = cta_range(a.TQ, a.G);
  const int total = 2 * a.S;
  auto slot = [&](int st) { return smem + (size_t)(st % kSlots) * kSlotBytes; };
  auto kind_of = [&](int st) { return st < a.S ? 0 : 1; };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlots; ++i) tc::mbar_init(&pp.slot_full[i], kHalf);
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&pp.means_ready[i], 1);
      tc::mbar_init(&pp.means_free[i], 1);
    }
    pp.abort = 0;
    pp.flag = 1;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();

  if (threadIdx.x < kHalf) {
    // ------------------------------------------------- statistics warps
    for (int st = 0; st <= total; ++st) {
      if (st < total) {
        if (!tc::wait_bounded(&pp.slot_full[st % kSlots], (uint32_t)((st / kSlots) & 1), abort_cta, a.status, 42,
                              a.wait_limit))
          break;
        if (st < a.S) k_stats<D>(a, st, slot(st), rk, sp);
        else v_stats<D>(a, st - a.S, slot(st), rk, reinterpret_cast<float*>(sp));
        count_in(a, kind_of(st), st % a.S);
      }
      if (st >= 1) {
        const int pv = st - 1, kind = kind_of(pv), grp = pv % a.S, b = pv & 1;
        const bool ok = wait_group(a, kind, grp, &pp.flag) &&
                        tc::wait_bounded(&pp.means_free[b], (uint32_t)(((pv >> 1) & 1) ^ 1), abort_cta, a.status,
                                         43, a.wait_limit);
        if (ok) {
          if (kind == 0) k_means<D>(a, grp, mean_buf + b * kMaxSliceChunkD, list, &pp.cnt);
          else v_scales<D>(a, grp, mean_buf + b * kMaxSliceChunkD);
        } else if (threadIdx.x == 0) {
          pp.flag = 0;
        }
        bar_half(kBarStats);
        if (threadIdx.x == 0) tc::mbar_arrive(&pp.means_ready[b]);  // also on failure: the quant warps look at flag
        if (!ok) break;
      }
    }
  } else {
    // ------------------------------------------------------ quant warps
    issue_slices<D>(a, kind_of(0), 0, slot(0), rk);
    cp_async_arrive_noinc(&pp.slot_full[0]);
    for (int st = 0; st <= total; ++st) {
      if (st + 1 < total) {
        bar_half(kBarQ);  // every quant thread is done with the slot of step st-2
        issue_slices<D>(a, kind_of(st + 1), (st + 1) % a.S, slot(st + 1), rk);
        cp_async_arrive_noinc(&pp.slot_full[(st + 1) % kSlots]);
      }
      if (st < a.S) {
        uint4 qx[kQPieces];
        q_load<D>(a, st, rq, qx);
        q_quant<D>(a, st, rq, qx, redq, &pp.anyq);
      }
      if (st >= 1) {
        const int pv = st - 1, b = pv & 1;
        const bool ok = tc::wait_bounded(&pp.means_ready[b], (uint32_t)((pv >> 1) & 1), abort_cta, a.status, 44,
                                         a.wait_limit);
        if (!ok || !pp.flag) break;
        const float* mb = mean_buf + b * kMaxSliceChunkD;
        if (pv < a.S) k_quant<D>(a, pv, slot(pv), rk, mb, red, &pp.anyk);
        else v_quant<D>(a, pv - a.S, slot(pv), rk, mb);
        bar_half(kBarQ);
        if (threadIdx.x == kHalf) tc::mbar_arrive(&pp.means_free[b]);
      }
    }
    asm volatile("cp.async.wait_all;" ::: "memory");  // no copy may land after the CTA has left
  }
}

// SM count and cooperative-launch support of the current device (asked on
// every call: the runtime answers from its own cache, and devices of one
// process may differ).
bool device_info(int* sms, int* coop) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess) return false;
  return *sms > 0;
}

struct Plan {
  int G, g, S, cpc, cpcq;
};

// Resident CTAs per SM of the kernel for D (0 on failure).
int ctas_per_sm(int D) {
  const void* fn = D == 128 ? reinterpret_cast<const void*>(prepass_resident_kernel<128>)
                            : reinterpret_cast<const void*>(prepass_resident_kernel<64>);
  int nb = 0;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, fn, kRThreads, kSmemBytes) != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  return std::min(nb, kCtasPerSm);
}

// The shape's partition for `slots` resident CTAs; false when one CTA's
// slice would not fit a slot (more than kMaxSliceChunkD chunks x channels).
bool make_plan(int B, int N, int H, int D, int slots, Plan* p) {
  const long long T64 = ceil_div(N, kKTile), TQ = (long long)ceil_div(N, kQTile) * (kQTile / kKTile);
  const long long U = (long long)B * H;
  const int G = (int)std::min<long long>(slots, T64);
  if (G <= 0) return false;
  const long long cpc = (T64 + G - 1) / G, cpcq = (TQ + G - 1) / G;
  const long long span = std::max(cpc, cpcq) * D;
  if (span > kMaxSliceChunkD) return false;
  p->G = G;
  p->cpc = (int)cpc;
  p->cpcq = (int)cpcq;
  p->g = (int)std::min<long long>(U, kMaxSliceChunkD / span);
  p->S = (int)((U + p->g - 1) / p->g);
  return true;
}

template <int D>
int resident(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N, int H,
             const FusedOut& o, const Plan& pl, cudaStream_t s) {
  ResArgs a;
  a.q = static_cast<const uint16_t*>(q.data);
  a.k = static_cast<const uint16_t*>(k.data);
  a.v = static_cast<const uint16_t*>(v.data);
  a.qsb = q.stride_b; a.qsn = q.stride_n; a.qsh = q.stride_h;
  a.ksb = k.stride_b; a.ksn = k.stride_n; a.ksh = k.stride_h;
  a.vsb = v.stride_b; a.vsn = v.stride_n; a.vsh = v.stride_h;
  a.N = N; a.H = H; a.U = B * H;
  a.Nq = ceil_div(N, kQTile) * kQTile;
  a.T64 = ceil_div(N, kKTile);
  a.Nk = a.T64 * kKTile;
  a.TQ = a.Nq / kKTile;
  a.G32 = ceil_div(N, kQGroup);
  a.G = pl.G; a.g = pl.g; a.S = pl.S; a.cpc = pl.cpc; a.cpcq = pl.cpcq;
  int l2 = 0;
  while ((1 << l2) < a.T64) ++l2;
  a.log2t = l2;
  a.q8 = o.q8; a.q_scale = o.q_scale; a.k8 = o.k8; a.k_scale = o.k_scale; a.k_mean = o.k_mean;
  a.v8 = o.v8; a.v_scale = o.v_scale;
  a.k_part = o.k_part;
  const size_t UD = (size_t)a.U * D;
  char* sync = reinterpret_cast<char*>(o.sync);
  a.k_sum = reinterpret_cast<double*>(sync);
  a.k_hi = reinterpret_cast<int*>(sync + UD * 8);
  a.k_lov = a.k_hi + UD;
  a.v_amax = a.k_lov + UD;
  a.arrive = a.v_amax + UD;
  a.abort_flag = a.arrive + 2 * (size_t)a.U;
  a.status = o.status;
  a.wait_limit = o.wait_limit;
  a.stall_unit = o.stall_unit;
  if (cudaMemsetAsync(o.sync, 0, prepass_sync_bytes(B, H, D), s) != cudaSuccess) return SAGE_ERR_CUDA;
  const void* fn = reinterpret_cast<const void*>(prepass_resident_kernel<D>);
  void* args[] = {&a};
  if (cudaLaunchCooperativeKernel(fn, dim3(pl.G), dim3(kRThreads), args, kSmemBytes, s) != cudaSuccess)
    return SAGE_ERR_CUDA;
  return SAGE_OK;
}

}  // namespace

size_t prepass_sync_bytes(int B, int H, int D) {
  const size_t U = (size_t)B * H;
  return U * D * (sizeof(double) + 3 * sizeof(int)) + (2 * U + 4) * sizeof(int);
}

// Resident CTA slots of the current device for D, or 0 when the kernel
// cannot run there (no cooperative launch, or no room for a CTA).
int resident_slots(int D) {
  int sms = 0, coop = 0;
  if ((D != 64 && D != 128) || !device_info(&sms, &coop) || !coop) return 0;
  return sms * ctas_per_sm(D);
}

bool prepass_fused_fits(int B, int N, int H, int D) {
  const int slots = resident_slots(D);
  Plan p;
  return slots > 0 && make_plan(B, N, H, D, slots, &p);
}

int launch_prepass_fused(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N,
                         int H, int D, const FusedOut& o, cudaStream_t s) {
  const int slots = resident_slots(D);
  Plan p;
  if (slots <= 0 || !make_plan(B, N, H, D, slots, &p)) return SAGE_ERR_UNSUPPORTED;
  if (D == 128) return resident<128>(q, k, v, B, N, H, o, p, s);
  return resident<64>(q, k, v, B, N, H, o, p, s);
}

}  // namespace sage
