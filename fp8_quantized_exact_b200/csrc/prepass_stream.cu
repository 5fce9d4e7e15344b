// Streaming prepass: K channel mean, Q/K INT8 and V E4M3 quantisation in one
// persistent launch whose work list puts the statistics of every head before
// its codes, so that the codes re-read K and V from L2 instead of HBM.
//
// Operation: the steps and rounding of the separate prepass kernels ("Sage2
// Blackwell Mainloop", sections "Decision" and "Existing Contract"), in one
// producer launch as the pages' P1/P2 producer fusions do ("Sage2 Blackwell
// Mainloop", section "Completed P1 And P2").  Bytes and scales equal those of
// the separate kernels.
//
// The work list.  An item is a 64-token tile of one head (unit u = b*H + h)
// and one of five kinds:
//   SK  K statistics: the FP64 token-order sum of the 64-token chunk, for
//       every channel;
//   SV  V statistics: the absolute maximum of every channel;
//   QQ  Q codes and scales (one 64-row block, two 32-row groups);
//   CK  K codes and scale of x - mean (one 64-row block);
//   CV  V codes (E4M3, transposed into channel rows).
// Persistent CTAs take items in list order from a global counter, one at a
// time or four consecutive ones when every CTA has many.  Round r of the
// list holds SK(r), SV(r), QQ(r) and, R heads behind, CK(r-R), CV(r-R).  A
// CTA counts a finished SK (SV) item in for its head with a release (a fence
// and a reduction), deferred until the loads of its next item are under way
// so that the fence's wait overlaps them.  A CK (CV) item waits (bounded)
// until all of its head's SK (SV) items are counted in and forms the K means
// (reads the V amax) itself from the accumulated statistics; the CTA keeps
// them for its next items of the same head.  A CTA only ever waits for items
// that come earlier in the list, which running CTAs have already taken and
// count in before their next wait, and SK, SV and QQ items wait for nothing,
// so every wait ends.  The host picks R so that about two grids' worth of
// items lie between a head's statistics and its codes: by then the
// statistics are done, and R heads of Q, K and V (a few tens of MB at the
// sizes used here, against 126 MB of L2) have passed through L2 since the
// head's K and V were read.
//
// The K mean is the FP64 sum of the FP64 chunk partials in chunk order,
// divided by N in FP64 and rounded once to FP32.  A nonzero partial p is a
// multiple of 2^lo(p) and below 2^(hi(p)+1) in magnitude; with lo and hi the
// minimum and maximum over a channel's chunks, every sum of partials is exact
// in FP64 when ceil(log2 T64) + hi - lo <= 52, and then any order of the
// additions gives the chunk-order sum bit for bit.  So each SK item adds its
// partial into an FP64 accumulator with an atomic add and publishes hi and
// lo with atomic maxima; a CK item takes the mean of a channel within the
// bound from the accumulator.  For channels outside it, the first CK item of
// the head to need them claims the head, adds the partials (kept in k_part)
// in chunk order, stores those means and publishes them; the other CK items
// of the head wait for that.
#include <algorithm>

#include "prepass_codes.cuh"

namespace sage {
namespace {

constexpr int kSThreads = 128;
constexpr int kSCtasPerSm = 6;
constexpr int kTok = 64;  // tokens of one item
enum : int { kSK = 0, kSV = 1, kQQ = 2, kCK = 3, kCV = 4 };

struct StreamArgs {
  const uint16_t *q, *k, *v;
  int64_t qsb, qsn, qsh, ksb, ksn, ksh, vsb, vsn, vsh;
  int N, H, U, Nq, Nk, T64, G32;
  int I;            // items of one kind per head: Nq / 64 (K and V items past T64 do nothing)
  int R;            // heads between a head's statistics and its codes
  int batch;        // consecutive items taken per work-list access (1 or 4)
  long long total;  // 5 * U * I
  int log2t;        // ceil(log2 T64)
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
  int* done;       // [2][U] zeroed: SK, SV items counted in
  int* fb_claim;   // [U] zeroed: 1 once a CK item has taken on the head's chunk-order means
  int* fb_ready;   // [U] zeroed: 1 once those means are stored
  int* abort_flag; // [1] zeroed
  unsigned long long* next;  // [1] zeroed: the work-list head
  DeviceStatus* status;
  long long wait_limit;
  int stall_unit;  // test hook: the first SK item of this head is never counted in (-1: none)
};

struct Item {
  int kind, u, part;
};

// Item j of the list of U heads, I tiles per kind and head, lag R (see the
// header comment for the order).  Host and device: the host export of the
// list is what the tests check.
__host__ __device__ __forceinline__ Item item_at(long long U, long long I, long long R, long long j) {
  const long long seg = j / I;
  Item it;
  it.part = (int)(j - seg * I);
  if (seg < 3 * (R < U ? R : U)) {
    it.kind = (int)(seg % 3);
    it.u = (int)(seg / 3);
  } else if (R < U && seg < 3 * R + 5 * (U - R)) {
    const long long s = seg - 3 * R;
    const int r = (int)(R + s / 5), k = (int)(s % 5);
    it.kind = k;
    it.u = k < 3 ? r : r - (int)R;
  } else {
    const long long s = seg - (R < U ? 3 * R + 5 * (U - R) : 3 * U);
    it.kind = kCK + (int)(s % 2);
    it.u = (int)((R < U ? U - R : 0) + s / 2);
  }
  return it;
}

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ uint32_t max_bf16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));  // a NaN operand yields the other
  return d;
}

// Bounded wait (thread 0) until a head's counter or flag reaches `target`.
// On timeout the status word records SAGE_ERR_TIMEOUT with `where`, and the
// abort flag stops the other CTAs at their next item.
__device__ bool wait_count(const StreamArgs& a, const int* flag, int target, int where) {
  const long long t0 = clock64();
  for (unsigned it = 0;; ++it) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v >= target) return true;
    if (*reinterpret_cast<volatile int*>(a.abort_flag)) return false;
    if (clock64() - t0 > a.wait_limit) {
      if (atomicCAS(&a.status->code, 0, (int)SAGE_ERR_TIMEOUT) == 0) {
        a.status->where = where;
        a.status->block = (int)blockIdx.x;
      }
      atomicExch(a.abort_flag, 1);
      return false;
    }
    __nanosleep(it < 8 ? 32 : 256);
  }
}

__device__ __forceinline__ void publish(int* flag) {
  __threadfence();
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(flag), "r"(1) : "memory");
}

// The deferred count of thread 0's previous SK or SV item: the barrier at
// the end of that item ordered all of its stores and atomics before this
// fence (cumulativity), so the reduction is seen only after them.  Called
// once the current item's loads are issued, before any wait.
__device__ __forceinline__ void settle(int*& pend) {
  if (threadIdx.x == 0 && pend) {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
    asm volatile("red.relaxed.gpu.global.add.s32 [%0], 1;" ::"l"(pend) : "memory");
    pend = nullptr;
  }
}

// Issues the copies of tokens [n0, n0 + 64) of one head's rows into the tile
// (rows past N zero-filled) as one cp.async group.  The 16-byte piece k of row r goes to
// position k ^ (2 * ((r >> 4) & 3)) of the row, so that the V code runs (16
// tokens of one channel pair per lane, four runs per warp) read 32 distinct
// banks; reads along a row stay conflict-free under any such permutation.
template <int D>
__device__ __forceinline__ void stage(const uint16_t* hp, int64_t sn, int n0, int N, uint32_t ts0) {
  constexpr int SEG = D / 8, COPIES = kTok * SEG / kSThreads;
#pragma unroll
  for (int i = 0; i < COPIES; ++i) {
    const int idx = threadIdx.x + kSThreads * i;
    const int r = idx / SEG, k = idx % SEG;
    const bool valid = n0 + r < N;
    cp_async_16_zfill(ts0 + (uint32_t)((r * SEG + (k ^ (2 * ((r >> 4) & 3)))) * 16),
                      valid ? hp + (int64_t)(n0 + r) * sn + k * 8 : hp, valid);
  }
  cp_async_commit();
}

__device__ __forceinline__ void staged() {
  cp_async_wait<0>();
  __syncthreads();
}

// ------------------------------------------------------------------- SK
// Thread t < D takes channel t of the chunk.
template <int D>
__device__ void do_sk(const StreamArgs& a, int u, int c, const uint8_t* tile) {
  constexpr int SEG = D / 8;
  const int d = threadIdx.x;
  if (d >= D || c >= a.T64) return;
  const int k = d >> 3, e = (d & 7) * 2;
  double p = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // (r >> 4) & 3 == q for rows 16q .. 16q + 15
    const uint8_t* base = tile + ((k ^ (2 * q)) << 4) + e;
    uint16_t w[16];  // the 16 loads first, so that the chain waits on one of them only
#pragma unroll
    for (int j = 0; j < 16; ++j) w[j] = *reinterpret_cast<const uint16_t*>(base + (16 * q + j) * SEG * 16);
#pragma unroll
    for (int j = 0; j < 16; ++j) p = __dadd_rn(p, (double)bf16_bits_to_f32(w[j]));  // token order; pad rows are zeros
  }
  a.k_part[((size_t)u * a.T64 + c) * D + d] = p;
  if (p != 0.0) {
    int ph, pl;
    partial_bits(p, ph, pl);
    const size_t at = (size_t)u * D + d;
    atomicAdd(a.k_sum + at, p);
    atomicMax(a.k_hi + at, kExpBias + ph);
    atomicMax(a.k_lov + at, kExpBias - pl);
  }
}

// The K means of head u into km_s[D] (all threads; after the head's SK
// items are all counted in).  Channels within the bound take theirs from the
// accumulator; for the others the chunk-order sums are formed once per head
// (by the CK item that claims them) and read back.  CK items of block 0
// store the means.
template <int D>
__device__ bool k_means(const StreamArgs& a, int u, bool store, float* km_s, int* list, int* s_cnt, int* s_flag) {
  const int t = threadIdx.x;
  if (t == 0) *s_cnt = 0;
  __syncthreads();
  for (int d = t; d < D; d += kSThreads) {
    const size_t at = (size_t)u * D + d;
    const int hi = __ldcg(a.k_hi + at) - kExpBias, lov = __ldcg(a.k_lov + at);
    if (lov == 0 || partials_exact(a.log2t, hi, kExpBias - lov)) {
      km_s[d] = lov == 0 ? 0.0f : __double2float_rn(__ddiv_rn(__ldcg(a.k_sum + at), (double)a.N));
      if (store) a.k_mean[at] = km_s[d];
    } else {
      list[atomicAdd(s_cnt, 1)] = d;
    }
  }
  __syncthreads();
  const int nlist = *s_cnt;
  if (nlist == 0) return true;
  if (t == 0) *s_flag = atomicCAS(a.fb_claim + u, 0, 1) == 0;
  __syncthreads();
  const bool claimed = *s_flag != 0;
  __syncthreads();  // s_flag is written again below
  if (claimed) {
    // channels off the bound: the chunk partials added in chunk order, one
    // warp per channel (lanes load 32 chunks at a time; every lane adds the
    // same values in the same order)
    const int warp = t >> 5, lane = t & 31;
    for (int e = warp; e < nlist; e += kSThreads / 32) {
      const int d = list[e];
      const double* src = a.k_part + (size_t)u * a.T64 * D + d;
      double total = 0.0;
      double nxt = lane < a.T64 ? __ldcg(src + (size_t)lane * D) : 0.0;
      for (int c0 = 0; c0 < a.T64; c0 += 32) {
        const double cur = nxt;
        if (c0 + 32 + lane < a.T64) nxt = __ldcg(src + (size_t)(c0 + 32 + lane) * D);
        const int n = min(32, a.T64 - c0);
        for (int j = 0; j < n; ++j) total = __dadd_rn(total, __shfl_sync(0xffffffffu, cur, j));
      }
      if (lane == 0) {
        km_s[d] = __double2float_rn(__ddiv_rn(total, (double)a.N));
        a.k_mean[(size_t)u * D + d] = km_s[d];
      }
    }
    __syncthreads();
    if (t == 0) publish(a.fb_ready + u);
    return true;
  }
  if (t == 0) *s_flag = wait_count(a, a.fb_ready + u, 1, 47);
  __syncthreads();
  if (!*s_flag) return false;
  for (int e = t; e < nlist; e += kSThreads) km_s[list[e]] = __ldcg(a.k_mean + (size_t)u * D + list[e]);
  __syncthreads();
  return true;
}

// ------------------------------------------------------------------- SV
// Thread t takes piece t % SEG (8 channels) of rows t / SEG + RPT * i.
template <int D>
__device__ void do_sv(const StreamArgs& a, int u, int c, uint32_t* redw, int*& pend) {
  constexpr int SEG = D / 8, RPT = kSThreads / SEG, PER = kTok / RPT, W = D / 2;
  const int t = threadIdx.x, k = t % SEG, lane = t & 31, warp = t >> 5;
  const uint16_t* hp = a.v + (u / a.H) * a.vsb + (u % a.H) * a.vsh + k * 8;
  const int n0 = c * kTok + t / SEG;
  uint4 x[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int n = n0 + RPT * i;
    x[i] = n < a.N ? ldg16(hp + (int64_t)n * a.vsn) : make_uint4(0, 0, 0, 0);
  }
  settle(pend);
  uint32_t m[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    m[0] = max_bf16x2(m[0], x[i].x & 0x7FFF7FFFu);
    m[1] = max_bf16x2(m[1], x[i].y & 0x7FFF7FFFu);
    m[2] = max_bf16x2(m[2], x[i].z & 0x7FFF7FFFu);
    m[3] = max_bf16x2(m[3], x[i].w & 0x7FFF7FFFu);
  }
#pragma unroll
  for (int o = SEG; o < 32; o <<= 1)
#pragma unroll
    for (int w = 0; w < 4; ++w) m[w] = max_bf16x2(m[w], __shfl_xor_sync(0xffffffffu, m[w], o));
  if (lane < SEG)
#pragma unroll
    for (int w = 0; w < 4; ++w) redw[warp * W + 4 * k + w] = m[w];  // word 4k+w: channels 8k+2w, +1
  __syncthreads();
  if (t < W) {
    uint32_t mm = redw[t];
#pragma unroll
    for (int w = 1; w < kSThreads / 32; ++w) mm = max_bf16x2(mm, redw[w * W + t]);
    // the amax of non-negative floats is exact in any order, and their bit
    // patterns order as integers
    const uint32_t lo = mm << 16, hi = mm & 0xFFFF0000u;
    int* dst = a.v_amax + (size_t)u * D + 2 * t;
    if (lo) atomicMax(dst, (int)lo);
    if (hi) atomicMax(dst + 1, (int)hi);
  }
}

// ------------------------------------------------------------------- QQ
// The 64-row block `blk` (two 32-row groups, each with its own scale);
// thread t holds 16-byte segments t + 128 i of the block, its first PER/2 in
// group 0.  Pad rows get zero codes, pad groups no scale.
template <int D>
__device__ void do_qq(const StreamArgs& a, int u, int blk, uint32_t* redb, float* redf, int*& pend) {
  constexpr int SEG = D / 8, PER = 2 * kQGroup * SEG / kSThreads;
  const int t = threadIdx.x, wl = t >> 5, lane = t & 31;
  const int r0 = blk * 2 * kQGroup;
  const int col = (t % SEG) * 8;
  const uint16_t* hp = a.q + (u / a.H) * a.qsb + (u % a.H) * a.qsh + col;
  uint4 xr[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int row = r0 + (t + kSThreads * i) / SEG;
    xr[i] = row < a.N ? ldg16(hp + (int64_t)row * a.qsn) : make_uint4(0, 0, 0, 0);
  }
  settle(pend);
  // amax as BF16 magnitude bits (NaN and inf above every finite value)
  uint32_t mb[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < PER; ++i) mb[i / (PER / 2)] = amax_bits8(xr[i], mb[i / (PER / 2)]);
#pragma unroll
  for (int g = 0; g < 2; ++g) mb[g] = __reduce_max_sync(0xffffffffu, halves_max(mb[g]));
  if (lane == 0) {
    redb[wl] = mb[0];
    redb[4 + wl] = mb[1];
  }
  __syncthreads();
  float am[2];
  bool finite[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    const uint32_t* rb = redb + 4 * g;
    mb[g] = max(max(rb[0], rb[1]), max(rb[2], rb[3]));
    finite[g] = mb[g] < 0x7F80u;
    am[g] = __uint_as_float(mb[g] << 16);
  }
  if (!finite[0] || !finite[1]) {
    // NaN or inf in the block: the amax that ignores NaN (the reference form)
    float af[2] = {0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      float f[8];
      unpack_bf16x8(xr[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) af[i / (PER / 2)] = fmaxf(af[i / (PER / 2)], fabsf(f[j]));
    }
    af[0] = warp_max(af[0]);
    af[1] = warp_max(af[1]);
    if (lane == 0) {
      redf[wl] = af[0];
      redf[4 + wl] = af[1];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < 2; ++g) am[g] = fmaxf(fmaxf(redf[4 * g], redf[4 * g + 1]), fmaxf(redf[4 * g + 2], redf[4 * g + 3]));
  }
  float inv[2];
  bool fast[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    inv[g] = am[g] > 0.0f ? __fdiv_rn(127.0f, am[g]) : 0.0f;
    fast[g] = finite[g] && codes_fast(am[g], inv[g]);
    const int grp = 2 * blk + g;
    if (t == 0 && grp < a.G32) a.q_scale[(size_t)u * a.G32 + grp] = am[g] > 0.0f ? __fdiv_rn(am[g], 127.0f) : 0.0f;
  }
  int8_t* dst = a.q8 + ((size_t)u * a.Nq + r0) * D + col;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int r = (t + kSThreads * i) / SEG;
    const float iv = inv[i / (PER / 2)];
    float f[8];
    unpack_bf16x8(xr[i], f);  // pad rows were loaded as zeros: zero codes
    const uint2 o = fast[i / (PER / 2)] ? i8_codes8_fast(f, iv) : i8_codes8_ref(f, iv);
    *reinterpret_cast<uint2*>(dst + (size_t)r * D) = o;
  }
}

// ------------------------------------------------------------------- CK
// The 64-row block tb; x' = fl32(x - k_mean[d]).  The raw BF16 rows stay in
// registers between the amax pass and the code pass (x' is recomputed, the
// same single rounding).
template <int D>
__device__ bool do_ck(const StreamArgs& a, int u, int tb, uint32_t* redb, float* redf, float* km_s, int* km_u,
                      int* list, int* s_cnt, int* s_flag, int*& pend) {
  constexpr int SEG = D / 8, PER = kKTile * SEG / kSThreads;
  const int t = threadIdx.x, wl = t >> 5, lane = t & 31;
  const int col = (t % SEG) * 8;
  const uint16_t* hp = a.k + (u / a.H) * a.ksb + (u % a.H) * a.ksh + col;
  uint4 xr[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int row = tb * kKTile + (t + kSThreads * i) / SEG;
    xr[i] = row < a.N ? ldg16(hp + (int64_t)row * a.ksn) : make_uint4(0, 0, 0, 0);
  }
  settle(pend);
  if (*km_u != u || tb == 0) {  // the CTA's cached means are another head's (block 0 stores them)
    if (t == 0) *s_flag = wait_count(a, a.done + u, a.I, 45);  // the head's statistics
    __syncthreads();
    if (!*s_flag) return false;
    if (!k_means<D>(a, u, tb == 0, km_s, list, s_cnt, s_flag)) return false;
    if (t == 0) *km_u = u;
  }
  float km[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) km[j] = km_s[col + j];
  float amax = 0.0f;  // NaN-propagating
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int row = tb * kKTile + (t + kSThreads * i) / SEG;
    if (row < a.N) {
      float f[8];
      unpack_bf16x8(xr[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmax_nan(amax, fabsf(__fsub_rn(f[j], km[j])));
    }
  }
  // the bits of non-negative floats order as integers, NaN above inf
  uint32_t ab = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  if (lane == 0) redb[wl] = ab;
  __syncthreads();
  ab = max(max(redb[0], redb[1]), max(redb[2], redb[3]));
  const bool finite = ab < 0x7F800000u;
  amax = __uint_as_float(ab);
  if (!finite) {
    // NaN or inf in the block: the amax that ignores NaN (the reference form)
    float af = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int row = tb * kKTile + (t + kSThreads * i) / SEG;
      if (row < a.N) {
        float f[8];
        unpack_bf16x8(xr[i], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) af = fmaxf(af, fabsf(__fsub_rn(f[j], km[j])));
      }
    }
    af = warp_max(af);
    if (lane == 0) redf[wl] = af;
    __syncthreads();
    amax = fmaxf(fmaxf(redf[0], redf[1]), fmaxf(redf[2], redf[3]));
  }
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  const bool fast = finite && codes_fast(amax, inv);
  if (t == 0) a.k_scale[(size_t)u * a.T64 + tb] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  int8_t* dst = a.k8 + ((size_t)u * a.Nk + (size_t)tb * kKTile) * D + col;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int r = (t + kSThreads * i) / SEG;
    uint2 o = make_uint2(0u, 0u);  // pad rows get zero codes
    if (tb * kKTile + r < a.N) {
      float f[8], x[8];
      unpack_bf16x8(xr[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __fsub_rn(f[j], km[j]);
      o = fast ? i8_codes8_fast(x, inv) : i8_codes8_ref(x, inv);
    }
    *reinterpret_cast<uint2*>(dst + (size_t)r * D) = o;
  }
  return true;
}

// ------------------------------------------------------------------- CV
// From the staged chunk c: each thread takes two adjacent channels of 16
// consecutive tokens (one 4-byte shared load per token gives both), converts
// them to E4M3 (two tokens per conversion, the earlier token in the low
// byte, so token t is byte t of the channel's row) and writes one 16-byte
// vector per channel; a warp writes 16 channels x 64 contiguous bytes.
template <int D>
__device__ void do_cv(const StreamArgs& a, int u, int c, const uint8_t* tb, const float* vam_s) {
  constexpr int SEG = D / 8, RUNS = (D / 2) * (kTok / 16) / kSThreads;
  const int n0 = c * kTok;
#pragma unroll
  for (int i = 0; i < RUNS; ++i) {
    const int idx = threadIdx.x + kSThreads * i;
    const int q = idx & 3, cp = (idx >> 2) & 7, pg = idx >> 5;
    const int t0 = 16 * q;               // first token of the run; (t >> 4) & 3 == q
    const int c0 = pg * 16 + 2 * cp;     // channels c0, c0 + 1
    const int k = c0 >> 3;               // their piece
    const float a0 = vam_s[c0], a1 = vam_s[c0 + 1];
    const float i0 = a0 > 0.0f ? __fdiv_rn(448.0f, a0) : 0.0f;
    const float i1 = a1 > 0.0f ? __fdiv_rn(448.0f, a1) : 0.0f;
    if (c == 0 && q == 0) {  // the channels' scales, once per head
      a.v_scale[(size_t)u * D + c0] = a0 > 0.0f ? __fdiv_rn(a0, 448.0f) : 0.0f;
      a.v_scale[(size_t)u * D + c0 + 1] = a1 > 0.0f ? __fdiv_rn(a1, 448.0f) : 0.0f;
    }
    const uint8_t* col = tb + ((k ^ (2 * q)) << 4) + ((c0 & 7) << 1);
    uint32_t wa[4], wc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + 4 * j;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) w[e] = *reinterpret_cast<const uint32_t*>(col + (t + e) * SEG * 16);
      const uint32_t alo = e4m3x2(__fmul_rn(__uint_as_float(w[0] << 16), i0), __fmul_rn(__uint_as_float(w[1] << 16), i0));
      const uint32_t ahi = e4m3x2(__fmul_rn(__uint_as_float(w[2] << 16), i0), __fmul_rn(__uint_as_float(w[3] << 16), i0));
      const uint32_t clo = e4m3x2(__fmul_rn(__uint_as_float(w[0] & 0xFFFF0000u), i1),
                                  __fmul_rn(__uint_as_float(w[1] & 0xFFFF0000u), i1));
      const uint32_t chi = e4m3x2(__fmul_rn(__uint_as_float(w[2] & 0xFFFF0000u), i1),
                                  __fmul_rn(__uint_as_float(w[3] & 0xFFFF0000u), i1));
      wa[j] = a0 > 0.0f ? (alo | (ahi << 16)) : 0u;
      wc[j] = a1 > 0.0f ? (clo | (chi << 16)) : 0u;
    }
    uint8_t* dst = a.v8 + ((size_t)u * D + c0) * a.Nk + n0 + t0;
    *reinterpret_cast<uint4*>(dst) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
    *reinterpret_cast<uint4*>(dst + a.Nk) = make_uint4(wc[0], wc[1], wc[2], wc[3]);
  }
}

// ---------------------------------------------------------------- kernel
// Takes the first index of the next a.batch items (thread 0); -1 once the
// kernel aborts.
__device__ __forceinline__ long long take(const StreamArgs& a) {
  long long j = (long long)atomicAdd(a.next, (unsigned long long)a.batch);
  if (*reinterpret_cast<volatile int*>(a.abort_flag)) j = -1;
  return j;
}

// Each CTA works on one item at a time, a.batch consecutive items per access
// to the list; the next batch's index is fetched during the last item of the
// current one.  Items of a batch are done in list order, so a wait still
// only depends on items taken earlier.
template <int D>
__global__ void __launch_bounds__(kSThreads, kSCtasPerSm) prepass_stream_kernel(const __grid_constant__ StreamArgs a) {
  __shared__ __align__(16) uint4 tile[kTok * D / 8];  // 64 rows of K or V
  __shared__ uint32_t redw[(kSThreads / 32) * (D / 2)];
  __shared__ uint32_t redb[8];
  __shared__ float redf[8];
  __shared__ float km_s[D];   // K means of head km_u
  __shared__ float vam_s[D];  // V channel amax of head vam_u
  __shared__ int list[D];
  __shared__ long long s_next;
  __shared__ int s_flag, s_cnt, km_u, vam_u;
  __shared__ Item s_it;
  const uint32_t ts0 = smem_u32(tile);
  const uint8_t* tb = reinterpret_cast<const uint8_t*>(tile);
  int* pend = nullptr;  // thread 0: the count its previous SK or SV item still owes
  // the mainloop that follows may start its set-up (it waits for this grid
  // to complete before it reads anything written here)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (threadIdx.x == 0) {
    s_next = take(a);
    km_u = -1;
    vam_u = -1;
  }
  __syncthreads();
  long long j = s_next;
  int left = a.batch;  // items of the current batch from j on
  while (j >= 0 && j < a.total) {
    long long jn = -1;
    if (threadIdx.x == 0 && left == 1) jn = take(a);  // used after this item
    if (threadIdx.x == 0) s_it = item_at(a.U, a.I, a.R, j);
    __syncthreads();
    const Item it = s_it;
    const int b = it.u / a.H, h = it.u % a.H;
    bool ok = true;
    if (it.kind == kSK || it.kind == kSV) {
      if (it.part < a.T64) {
        if (it.kind == kSK) {
          stage<D>(a.k + b * a.ksb + h * a.ksh, a.ksn, it.part * kTok, a.N, ts0);
          settle(pend);
          staged();
          do_sk<D>(a, it.u, it.part, tb);
        } else {
          do_sv<D>(a, it.u, it.part, redw, pend);
        }
      }
      settle(pend);
      __syncthreads();  // the item's stores and atomics come before its count
      if (threadIdx.x == 0 && !(it.kind == kSK && it.part == 0 && it.u == a.stall_unit))
        pend = a.done + (it.kind == kSK ? 0 : a.U) + it.u;
    } else if (it.kind == kQQ) {
      do_qq<D>(a, it.u, it.part, redb, redf, pend);
    } else if (it.part < a.T64) {
      if (it.kind == kCK) {
        ok = do_ck<D>(a, it.u, it.part, redb, redf, km_s, &km_u, list, &s_cnt, &s_flag, pend);
      } else {
        stage<D>(a.v + b * a.vsb + h * a.vsh, a.vsn, it.part * kTok, a.N, ts0);
        settle(pend);
        if (vam_u != it.u) {  // the CTA's cached amax are another head's
          if (threadIdx.x == 0) s_flag = wait_count(a, a.done + a.U + it.u, a.I, 46);  // the head's statistics
          __syncthreads();
          ok = s_flag != 0;
          if (ok)
            for (int d = threadIdx.x; d < D; d += kSThreads) vam_s[d] = __int_as_float(__ldcg(a.v_amax + (size_t)it.u * D + d));
          if (threadIdx.x == 0) vam_u = it.u;
        }
        staged();
        if (ok) do_cv<D>(a, it.u, it.part, tb, vam_s);
      }
    } else {
      settle(pend);
    }
    if (left > 1) {
      __syncthreads();  // the tile and the scratch are free again
      if (!ok) break;
      ++j;
      --left;
      continue;
    }
    if (threadIdx.x == 0) s_next = jn;
    __syncthreads();  // the tile, the scratch, s_flag and s_next are consistent again
    if (!ok) break;
    j = s_next;
    left = a.batch;
    __syncthreads();  // s_next is rewritten by the next batch
  }
  settle(pend);
  asm volatile("cp.async.wait_all;" ::: "memory");  // no copy may land after the CTA has left
}

// Heads between a head's statistics and its codes: the fewest that put
// about two grids' worth of items between them (5R + 2 item runs of I).
int pick_lag(int U, int I, long long grid) {
  int R = 1;
  while (R < U && (long long)(5 * R + 2) * I < 2 * grid) ++R;
  return R;
}

template <int D>
int stream(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N, int H,
           const FusedOut& o, cudaStream_t s) {
  int dev = 0, sms = 0, occ = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, prepass_stream_kernel<D>, kSThreads, 0) != cudaSuccess ||
      sms <= 0 || occ <= 0) {
    cudaGetLastError();
    return SAGE_ERR_CUDA;
  }
  StreamArgs a;
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
  a.G32 = ceil_div(N, kQGroup);
  a.I = a.Nq / kTok;
  a.total = 5LL * a.U * a.I;
  const int grid = (int)std::min<long long>((long long)sms * std::min(occ, kSCtasPerSm), a.total);
  // batches of four when every CTA has many items (fewer accesses to the
  // list counter); single items otherwise, so that all CTAs get work
  a.batch = a.total >= 16LL * grid ? 4 : 1;
  a.R = pick_lag(a.U, a.I, grid);
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
  a.done = a.v_amax + UD;
  a.fb_claim = a.done + 2 * (size_t)a.U;
  a.fb_ready = a.fb_claim + a.U;
  a.abort_flag = a.fb_ready + a.U;
  const size_t next_off = (UD * 20 + (4 * (size_t)a.U + 1) * sizeof(int) + 7) & ~(size_t)7;
  a.next = reinterpret_cast<unsigned long long*>(sync + next_off);
  a.status = o.status;
  a.wait_limit = o.wait_limit;
  a.stall_unit = o.stall_unit;
  if (cudaMemsetAsync(o.sync, 0, prepass_sync_bytes(B, H, D), s) != cudaSuccess) return SAGE_ERR_CUDA;
  prepass_stream_kernel<D><<<grid, kSThreads, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

int prepass_stream_list(int B, int N, int H, int grid, int* lag, long long n, int* items) {
  const int U = B * H, I = ceil_div(N, kQTile) * kQTile / kTok;
  if (5LL * U * I != n || grid <= 0) return SAGE_ERR_INVALID_ARG;
  const int R = pick_lag(U, I, grid);
  if (lag) *lag = R;
  for (long long j = 0; j < n; ++j) {
    const Item it = item_at(U, I, R, j);
    items[3 * j] = it.kind;
    items[3 * j + 1] = it.u;
    items[3 * j + 2] = it.part;
  }
  return SAGE_OK;
}

size_t prepass_sync_bytes(int B, int H, int D) {
  // per channel: an FP64 sum and three ints; per head: four ints (counts and
  // claims); then the abort flag and an 8-byte work-list head
  const size_t U = (size_t)B * H;
  return U * D * (sizeof(double) + 3 * sizeof(int)) + (4 * U + 4) * sizeof(int) + 8;
}

int launch_prepass_stream(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N,
                          int H, int D, const FusedOut& o, cudaStream_t s) {
  if (D == 128) return stream<128>(q, k, v, B, N, H, o, s);
  if (D == 64) return stream<64>(q, k, v, B, N, H, o, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
