// Single-launch prepass: K channel mean, Q/K INT8 and V E4M3 quantisation in
// one persistent kernel, with each head's K and V read from HBM once and
// re-read from L2 for the quantisation.
//
// Operation: the same steps and rounding as the separate prepass kernels
// ("Sage2 Blackwell Mainloop", sections "Decision" and "Existing
// Contract"); the fusion of the producers follows the pages' P1/P2 producer
// fusions ("Sage2 Blackwell Mainloop", section "Completed P1 And P2").  The
// bytes and scales are identical to the separate kernels: the FP64 K sums
// run in token order inside each 64-token chunk and the chunk partials are
// added in chunk order by one thread per channel.
//
// Work is handed out by a global ticket in head-major order, in slots; slot
// s holds, for head s, nS statistics items (CPI chunks of 64 tokens each:
// FP64 K sums and V amax partials; the CTA that completes the head's last
// chunk reduces the partials to k_mean, v_amax and v_scale and raises the
// head flag) and nQ Q items (16 groups of 32 rows each), and for head
// s - kLookahead its nS K/V items (CPI chunks: wait for the head flag, then
// K smoothing and INT8 K, E4M3 V stored transposed).  The lookahead gives
// the statistics of a head time to finish before its K/V items are taken,
// while the K and V of the heads in flight (about 20 MB each) stay in L2.
// A K/V item only ever waits for statistics items with smaller tickets,
// which running CTAs have already claimed and finish without waiting, so
// the waits always end; they are bounded all the same (the status word
// records SAGE_ERR_TIMEOUT and the item is skipped).
#include <algorithm>

#include "sage_common.cuh"

namespace sage {
namespace {

constexpr int kThreadsP = 256;
constexpr int kQPerItem = 16;  // 32-row Q groups per Q item (two per warp)
constexpr int kLookahead = 2;  // heads between a head's statistics and its K/V items

__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ld16(const uint16_t* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

__device__ __forceinline__ uint32_t code_i8(float x, float inv) {
  int r = __float2int_rn(__fmul_rn(x, inv));
  r = max(-127, min(127, r));
  return static_cast<uint32_t>(r) & 0xFFu;
}

struct FusedArgs {
  const uint16_t *q, *k, *v;
  int64_t qsb, qsn, qsh, ksb, ksn, ksh, vsb, vsn, vsh;
  int B, N, H, Nq, Nk, T64, G32, Gq;  // Gq: 32-row groups of the padded Q (Nq / 32)
  int nS, nQ, per_head;              // items per head: nS stats, nQ Q, nS K/V
  int BH;
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  float* k_mean;
  uint8_t* v8;
  float* v_scale;
  float* v_amax;
  double* k_part;
  float* v_part;
  int* ticket;     // [1]
  int* head_done;  // [B*H] chunks whose statistics are written
  int* head_flag;  // [B*H] 1 once k_mean / v_amax of the head are written
  DeviceStatus* status;
  long long wait_limit;
};

// ------------------------------------------------------------ statistics
// Threads 0..127: K sums, threads 128..255: V amax; D/8 threads per chunk,
// each owning 8 consecutive channels.
template <int D>
__device__ void stats_item(const FusedArgs& a, int bh, int c0, int c1) {
  constexpr int TPC = D / 8;
  const int half = threadIdx.x >> 7, t = threadIdx.x & 127;
  const int chunk = c0 + t / TPC, col = (t % TPC) * 8;
  const int b = bh / a.H, h = bh % a.H;
  if (chunk < c1) {
    const int n0 = chunk * kKTile, n1 = min(n0 + kKTile, a.N);
    const size_t o = ((size_t)bh * a.T64 + chunk) * D + col;
    if (half == 0) {
      double ks[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) ks[i] = 0.0;
      const uint16_t* kp = a.k + b * a.ksb + h * a.ksh + col;
#pragma unroll 16
      for (int n = n0; n < n1; ++n) {
        float f[8];
        unpack8(ld16(kp + n * a.ksn), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) ks[i] = __dadd_rn(ks[i], (double)f[i]);
      }
      double2* dst = reinterpret_cast<double2*>(a.k_part + o);
#pragma unroll
      for (int i = 0; i < 4; ++i) dst[i] = make_double2(ks[2 * i], ks[2 * i + 1]);
    } else {
      float vm[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) vm[i] = 0.0f;
      const uint16_t* vp = a.v + b * a.vsb + h * a.vsh + col;
#pragma unroll 16
      for (int n = n0; n < n1; ++n) {
        float f[8];
        unpack8(ld16(vp + n * a.vsn), f);
#pragma unroll
        for (int i = 0; i < 8; ++i) vm[i] = fmaxf(vm[i], fabsf(f[i]));
      }
      float4* dst = reinterpret_cast<float4*>(a.v_part + o);
      dst[0] = make_float4(vm[0], vm[1], vm[2], vm[3]);
      dst[1] = make_float4(vm[4], vm[5], vm[6], vm[7]);
    }
  }
  // count the chunks; the CTA that completes the head reduces it
  __shared__ int last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) last = atomicAdd(&a.head_done[bh], c1 - c0) + (c1 - c0) == a.T64;
  __syncthreads();
  if (!last) return;
  __threadfence();
  if (threadIdx.x < D) {
    const int d = threadIdx.x;
    // partials added in chunk order; loads fetched 16 ahead of the adds
    const double* src = a.k_part + (size_t)bh * a.T64 * D + d;
    double total = 0.0;
    for (int c0 = 0; c0 < a.T64; c0 += 16) {
      double x[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] = c0 + j < a.T64 ? __ldcg(src + (size_t)(c0 + j) * D) : 0.0;
#pragma unroll
      for (int j = 0; j < 16; ++j)
        if (c0 + j < a.T64) total = __dadd_rn(total, x[j]);
    }
    a.k_mean[(size_t)bh * D + d] = __double2float_rn(__ddiv_rn(total, (double)a.N));
  } else if (threadIdx.x >= 128 && threadIdx.x < 128 + D) {
    const int d = threadIdx.x - 128;
    const float* src = a.v_part + (size_t)bh * a.T64 * D + d;
    float am = 0.0f;
    for (int c0 = 0; c0 < a.T64; c0 += 16) {
      float x[16];
#pragma unroll
      for (int j = 0; j < 16; ++j) x[j] = c0 + j < a.T64 ? __ldcg(src + (size_t)(c0 + j) * D) : 0.0f;
#pragma unroll
      for (int j = 0; j < 16; ++j) am = fmaxf(am, x[j]);
    }
    a.v_amax[(size_t)bh * D + d] = am;
    a.v_scale[(size_t)bh * D + d] = am > 0.0f ? __fdiv_rn(am, 448.0f) : 0.0f;
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) atomicExch(&a.head_flag[bh], 1);
}

// ---------------------------------------------------------------------- Q
// One warp per 32-row group, two groups per warp; pad rows and pad groups
// of the padded Q get zero bytes.
template <int D>
__device__ void q_item(const FusedArgs& a, int bh, int g0) {
  constexpr int SEG = D / 8;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = bh / a.H, h = bh % a.H;
#pragma unroll 1
  for (int k = 0; k < 2; ++k) {
    const int g = g0 + 2 * warp + k;
    if (g >= a.Gq) break;
    const int r0 = g * kQGroup;
    uint4 x[SEG];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < SEG; ++i) {
      const int s = lane + 32 * i;
      const int row = r0 + s / SEG, col = (s % SEG) * 8;
      x[i] = row < a.N ? ld16(a.q + b * a.qsb + (int64_t)row * a.qsn + h * a.qsh + col) : make_uint4(0, 0, 0, 0);
      float f[8];
      unpack8(x[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
    }
    amax = warp_max(amax);
    const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    if (lane == 0 && g < a.G32) a.q_scale[(size_t)bh * a.G32 + g] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
    int8_t* dst = a.q8 + ((size_t)bh * a.Nq + r0) * D;
#pragma unroll
    for (int i = 0; i < SEG; ++i) {
      const int s = lane + 32 * i;
      const int row = s / SEG, col = (s % SEG) * 8;
      float f[8];
      unpack8(x[i], f);
      uint2 o;
      o.x = code_i8(f[0], inv) | code_i8(f[1], inv) << 8 | code_i8(f[2], inv) << 16 | code_i8(f[3], inv) << 24;
      o.y = code_i8(f[4], inv) | code_i8(f[5], inv) << 8 | code_i8(f[6], inv) << 16 | code_i8(f[7], inv) << 24;
      *reinterpret_cast<uint2*>(dst + (size_t)row * D + col) = o;
    }
  }
}

// -------------------------------------------------------------------- K/V
// Wait (bounded) for the head's statistics; returns false on timeout.
__device__ bool wait_head(const FusedArgs& a, int bh) {
  __shared__ int ok;
  if (threadIdx.x == 0) {
    const long long t0 = clock64();
    int f = 0;
    for (unsigned i = 0;; ++i) {
      asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(f) : "l"(a.head_flag + bh) : "memory");
      if (f) break;
      if (clock64() - t0 > a.wait_limit) break;
      __nanosleep(i < 16 ? 64 : 256);
    }
    ok = f;
    if (!f && atomicCAS(&a.status->code, 0, (int)SAGE_ERR_TIMEOUT) == 0) {
      a.status->where = 30;
      a.status->block = (int)blockIdx.x;
    }
  }
  __syncthreads();
  return ok != 0;
}

// K: 128 threads per 64-row chunk, two chunks at a time; x' = fl32(x - km).
// The raw BF16 chunks stay in registers between the amax and code passes.
template <int D>
__device__ void k_quant(const FusedArgs& a, int bh, int c0, int c1) {
  constexpr int SEG = D / 8;
  constexpr int PER = kKTile * SEG / 128;
  const int half = threadIdx.x >> 7, t = threadIdx.x & 127;
  const int b = bh / a.H, h = bh % a.H;
  const int col = (t % SEG) * 8;
  float km[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) km[j] = __ldcg(a.k_mean + (size_t)bh * D + col + j);
  __shared__ float red[8];
#pragma unroll 1
  for (int cb = c0; cb < c1; cb += 2) {
    const int chunk = cb + half;
    const bool live = chunk < c1;
    uint4 xr[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int row = chunk * kKTile + (t + 128 * i) / SEG;
      xr[i] = live && row < a.N ? ld16(a.k + b * a.ksb + (int64_t)row * a.ksn + h * a.ksh + col)
                                : make_uint4(0, 0, 0, 0);
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int row = chunk * kKTile + (t + 128 * i) / SEG;
      if (live && row < a.N) {
        float f[8];
        unpack8(xr[i], f);
#pragma unroll
        for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(__fsub_rn(f[j], km[j])));
      }
    }
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[4 * half], red[4 * half + 1]), fmaxf(red[4 * half + 2], red[4 * half + 3]));
    __syncthreads();
    if (live) {
      const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
      if (t == 0) a.k_scale[(size_t)bh * a.T64 + chunk] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
      int8_t* dst = a.k8 + ((size_t)bh * a.Nk + (size_t)chunk * kKTile) * D;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int r = (t + 128 * i) / SEG;
        uint2 o = make_uint2(0u, 0u);  // pad rows get zero codes
        if (chunk * kKTile + r < a.N) {
          float f[8], x[8];
          unpack8(xr[i], f);
#pragma unroll
          for (int j = 0; j < 8; ++j) x[j] = __fsub_rn(f[j], km[j]);
          o.x = code_i8(x[0], inv) | code_i8(x[1], inv) << 8 | code_i8(x[2], inv) << 16 | code_i8(x[3], inv) << 24;
          o.y = code_i8(x[4], inv) | code_i8(x[5], inv) << 8 | code_i8(x[6], inv) << 16 | code_i8(x[7], inv) << 24;
        }
        *reinterpret_cast<uint2*>(dst + (size_t)r * D + col) = o;
      }
    }
  }
}

// V: 128 tokens at a time staged in shared memory with 16-byte loads (the
// chunk index of a row XORed with bits 4-5 of its token, so that the column
// reads hit distinct banks); each thread then converts 16 consecutive tokens
// of one channel to E4M3 (token t in byte t of the channel's row) and writes
// them as one 16-byte vector.
constexpr int kVBlock = 2 * kKTile;

template <int D>
__device__ void v_quant(const FusedArgs& a, int bh, int c0, int c1) {
  constexpr int SEG = D / 8;
  constexpr int LOADS = kVBlock * SEG / kThreadsP;
  constexpr int RUNS = D * (kVBlock / 16) / kThreadsP;
  __shared__ __align__(16) uint4 tile[kVBlock * SEG];
  const int b = bh / a.H, h = bh % a.H;
  const uint16_t* vp = a.v + b * a.vsb + h * a.vsh;
  const float* am = a.v_amax + (size_t)bh * D;
  const uint16_t* ts = reinterpret_cast<const uint16_t*>(tile);
  const int tok1 = min(c1 * kKTile, a.Nk);  // end of this item's tokens (padded length)
#pragma unroll 1
  for (int n0 = c0 * kKTile; n0 < tok1; n0 += kVBlock) {
    __syncthreads();  // the previous block's column reads are done
    // staged in two rounds of loads, to stay within the registers
#pragma unroll
    for (int i0 = 0; i0 < LOADS; i0 += LOADS / 2) {
      uint4 x[LOADS / 2];
#pragma unroll
      for (int i = 0; i < LOADS / 2; ++i) {
        const int idx = threadIdx.x + kThreadsP * (i0 + i);
        const int r = idx / SEG, k = idx % SEG;
        x[i] = n0 + r < a.N ? ld16(vp + (int64_t)(n0 + r) * a.vsn + k * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int i = 0; i < LOADS / 2; ++i) {
        const int idx = threadIdx.x + kThreadsP * (i0 + i);
        const int r = idx / SEG, k = idx % SEG;
        tile[r * SEG + (k ^ ((r >> 4) & 3))] = x[i];
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < RUNS; ++i) {
      const int idx = threadIdx.x + kThreadsP * i;
      const int q = idx & 3, cl = (idx >> 2) & 7, rest = idx >> 5;
      const int cb = rest % SEG, hf = rest / SEG;
      const int t0 = hf * kKTile + 16 * q;
      if (n0 + hf * kKTile >= tok1) continue;
      const int ch = cb * 8 + cl;
      const float amx = __ldcg(am + ch);
      const float inv = amx > 0.0f ? __fdiv_rn(448.0f, amx) : 0.0f;
      const uint16_t* col = ts + (cb ^ q) * 8 + cl;
      uint32_t w[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = t0 + 4 * j;
        const uint32_t lo = e4m3x2(__fmul_rn(bf16_bits_to_f32(col[t * D]), inv),
                                   __fmul_rn(bf16_bits_to_f32(col[(t + 1) * D]), inv));
        const uint32_t hi = e4m3x2(__fmul_rn(bf16_bits_to_f32(col[(t + 2) * D]), inv),
                                   __fmul_rn(bf16_bits_to_f32(col[(t + 3) * D]), inv));
        w[j] = amx > 0.0f ? (lo | (hi << 16)) : 0u;
      }
      uint8_t* dst = a.v8 + ((size_t)bh * D + ch) * a.Nk + n0 + t0;
      *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreadsP, 2) prepass_fused_kernel(const FusedArgs a) {
  constexpr int CPI = 128 / (D / 8);  // chunks per statistics or K/V item
  __shared__ int item_s;
  // a slot of the ticket sequence: statistics and Q items of head s, then
  // the K/V items of head s - kLookahead (either part may be absent)
  const int total = (a.BH + kLookahead) * a.per_head;
  for (;;) {
    __syncthreads();
    if (threadIdx.x == 0) item_s = atomicAdd(a.ticket, 1);
    __syncthreads();
    const int item = item_s;
    if (item >= total) break;
    const int slot = item / a.per_head, r = item % a.per_head;
    if (r < a.nS + a.nQ) {
      const int bh = slot;
      if (bh >= a.BH) continue;
      if (r < a.nS) stats_item<D>(a, bh, r * CPI, min(a.T64, (r + 1) * CPI));
      else q_item<D>(a, bh, (r - a.nS) * kQPerItem);
    } else {
      const int bh = slot - kLookahead;
      if (bh < 0) continue;
      const int u = r - a.nS - a.nQ;
      if (!wait_head(a, bh)) continue;
      const int c0 = u * CPI, c1 = min(a.T64, (u + 1) * CPI);
      k_quant<D>(a, bh, c0, c1);
      v_quant<D>(a, bh, c0, c1);
    }
  }
}

// SM count of the current device (asked on every call: the runtime answers
// from its own cache, and devices of one process may differ)
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      n <= 0)
    n = 148;
  return n;
}

// Work items of one call: the kernel's ticket counter and its item count are
// int, and each CTA draws one ticket past the end before it leaves.
constexpr long long kMaxItems = 1LL << 30;

template <int D>
long long fused_items(int B, int N, int H) {
  constexpr int CPI = 128 / (D / 8);
  const long long T64 = ceil_div(N, kKTile), Gq = ceil_div(N, kQTile) * kQTile / kQGroup;
  const long long per_head = 2 * ((T64 + CPI - 1) / CPI) + (Gq + kQPerItem - 1) / kQPerItem;
  return ((long long)B * H + kLookahead) * per_head;
}

template <int D>
int fused(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N, int H,
          const FusedOut& o, cudaStream_t s) {
  constexpr int CPI = 128 / (D / 8);
  FusedArgs a;
  a.q = static_cast<const uint16_t*>(q.data);
  a.k = static_cast<const uint16_t*>(k.data);
  a.v = static_cast<const uint16_t*>(v.data);
  a.qsb = q.stride_b; a.qsn = q.stride_n; a.qsh = q.stride_h;
  a.ksb = k.stride_b; a.ksn = k.stride_n; a.ksh = k.stride_h;
  a.vsb = v.stride_b; a.vsn = v.stride_n; a.vsh = v.stride_h;
  a.B = B; a.N = N; a.H = H;
  a.Nq = ceil_div(N, kQTile) * kQTile;
  a.T64 = ceil_div(N, kKTile);
  a.Nk = a.T64 * kKTile;
  a.G32 = ceil_div(N, kQGroup);
  a.Gq = a.Nq / kQGroup;
  a.nS = ceil_div(a.T64, CPI);
  a.nQ = ceil_div(a.Gq, kQPerItem);
  a.per_head = 2 * a.nS + a.nQ;
  a.BH = B * H;
  a.q8 = o.q8; a.q_scale = o.q_scale; a.k8 = o.k8; a.k_scale = o.k_scale; a.k_mean = o.k_mean;
  a.v8 = o.v8; a.v_scale = o.v_scale; a.v_amax = o.v_amax; a.k_part = o.k_part; a.v_part = o.v_part;
  a.ticket = o.counters;
  a.head_done = o.counters + 1;
  a.head_flag = o.counters + 1 + B * H;
  a.status = o.status;
  a.wait_limit = o.wait_limit;
  if (cudaMemsetAsync(o.counters, 0, sizeof(int) * (1 + 2 * (size_t)B * H), s) != cudaSuccess) return SAGE_ERR_CUDA;
  const long long items = fused_items<D>(B, N, H);
  if (items > kMaxItems) return SAGE_ERR_UNSUPPORTED;
  const int grid = (int)std::min<long long>(items, 2LL * sm_count());
  prepass_fused_kernel<D><<<grid, kThreadsP, 0, s>>>(a);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

bool prepass_fused_fits(int B, int N, int H, int D) {
  if (D != 64 && D != 128) return false;
  return (D == 128 ? fused_items<128>(B, N, H) : fused_items<64>(B, N, H)) <= kMaxItems;
}

int launch_prepass_fused(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N,
                         int H, int D, const FusedOut& o, cudaStream_t s) {
  if (D == 128) return fused<128>(q, k, v, B, N, H, o, s);
  if (D == 64) return fused<64>(q, k, v, B, N, H, o, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
