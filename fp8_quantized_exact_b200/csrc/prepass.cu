// Prepass kernels: K channel mean, Q/K INT8 quantisation, V E4M3
// quantisation with a transposed store.  All are HBM-bound streaming
// kernels: 16-byte vector loads of the strided BF16 views, one pass per
// statistic, results written once.
//
// Operation defined by "Sage2 Blackwell Mainloop", section "Decision"
// (K mean/smoothing, Q quantization, K subtract-mean quantization, V
// transpose/pad/permute, V scale/FP8 quantization) and section "Existing
// Contract" (per-warp INT8 Q in 32-row groups, per-block INT8 K with 64-row
// blocks, FP8 V with a per-channel scale).  The exact rounding steps follow
// the readings stated in include/sage_b200.h.
#include "sage_common.cuh"

namespace sage {
namespace {

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// INT8 code of one product, round half to even, clamped to +-127.
__device__ __forceinline__ uint32_t i8_code(float x, float inv) {
  int r = __float2int_rn(__fmul_rn(x, inv));
  r = max(-127, min(127, r));
  return static_cast<uint32_t>(r) & 0xFFu;
}

// ------------------------------------------------------------------------
// Per 64-token chunk: FP64 sum of each K channel (tokens added in order) and
// the FP32 amax of each V channel.  One thread owns 8 consecutive channels
// of one chunk; D/8 threads per chunk; 128 threads per block.
template <int D, bool DO_K, bool DO_V>
__global__ void __launch_bounds__(128) chunk_stats_kernel(
    const uint16_t* __restrict__ k, int64_t ksb, int64_t ksn, int64_t ksh,
    const uint16_t* __restrict__ v, int64_t vsb, int64_t vsn, int64_t vsh, int N, int H, int T64,
    double* __restrict__ k_part, float* __restrict__ v_part) {
  constexpr int TPC = D / 8;
  constexpr int CPB = 128 / TPC;
  const int chunk = blockIdx.x * CPB + threadIdx.x / TPC;
  const int col = (threadIdx.x % TPC) * 8;
  const int h = blockIdx.y, b = blockIdx.z;
  if (chunk >= T64) return;
  const int n0 = chunk * kKTile;
  const int n1 = min(n0 + kKTile, N);
  double ks[8];
  float vm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) { ks[i] = 0.0; vm[i] = 0.0f; }
  const uint16_t* kp = k + b * ksb + h * ksh + col;
  const uint16_t* vp = v + b * vsb + h * vsh + col;
#pragma unroll 4
  for (int n = n0; n < n1; ++n) {
    if (DO_K) {
      float f[8];
      unpack_bf16x8(ldg16(kp + n * ksn), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) ks[i] = __dadd_rn(ks[i], (double)f[i]);
    }
    if (DO_V) {
      float f[8];
      unpack_bf16x8(ldg16(vp + n * vsn), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) vm[i] = fmaxf(vm[i], fabsf(f[i]));
    }
  }
  const size_t o = ((size_t)(b * H + h) * T64 + chunk) * D + col;
  if (DO_K) {
    double2* dst = reinterpret_cast<double2*>(k_part + o);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = make_double2(ks[2 * i], ks[2 * i + 1]);
  }
  if (DO_V) {
    float4* dst = reinterpret_cast<float4*>(v_part + o);
    dst[0] = make_float4(vm[0], vm[1], vm[2], vm[3]);
    dst[1] = make_float4(vm[4], vm[5], vm[6], vm[7]);
  }
}

// Chunk partials -> k_mean (partials added in chunk order, then one FP64
// division and one rounding to FP32) and V amax / v_scale.  One thread per
// (b, h, d).
template <bool DO_K, bool DO_V>
__global__ void reduce_stats_kernel(int N, int D, int T64, const double* __restrict__ k_part,
                                    float* __restrict__ k_mean, const float* __restrict__ v_part,
                                    float* __restrict__ v_scale, float* __restrict__ v_amax) {
  const int d = threadIdx.x;
  const size_t bh = blockIdx.x;
  if (d >= D) return;
  if (DO_K) {
    double total = 0.0;
    for (int c = 0; c < T64; ++c) total = __dadd_rn(total, k_part[(bh * T64 + c) * D + d]);
    k_mean[bh * D + d] = __double2float_rn(__ddiv_rn(total, (double)N));
  }
  if (DO_V) {
    float am = 0.0f;
    for (int c = 0; c < T64; ++c) am = fmaxf(am, v_part[(bh * T64 + c) * D + d]);
    v_amax[bh * D + d] = am;
    v_scale[bh * D + d] = am > 0.0f ? __fdiv_rn(am, 448.0f) : 0.0f;
  }
}

// ------------------------------------------------------------------------
// Q: one warp per 32-row group, four warps per 128-row block (the rows of a
// block are one mainloop query tile).  Pad rows and pad groups get zeros.
template <int D>
__global__ void __launch_bounds__(128) quant_q_kernel(const uint16_t* __restrict__ q, int64_t sb,
                                                      int64_t sn, int64_t sh, int N, int H, int Nq,
                                                      int G32, int8_t* __restrict__ q8,
                                                      float* __restrict__ q_scale) {
  constexpr int SEG = D / 8;  // 16-byte segments per row == segments per lane
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x * 4 + warp;
  const int h = blockIdx.y, b = blockIdx.z;
  const int r0 = g * kQGroup;
  uint4 x[SEG];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < SEG; ++i) {
    const int s = lane + 32 * i;
    const int row = r0 + s / SEG, col = (s % SEG) * 8;
    x[i] = row < N ? ldg16(q + b * sb + (int64_t)row * sn + h * sh + col) : make_uint4(0, 0, 0, 0);
    float f[8];
    unpack_bf16x8(x[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(f[j]));
  }
  amax = warp_max(amax);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  if (lane == 0 && g < G32)
    q_scale[(size_t)(b * H + h) * G32 + g] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  int8_t* dst = q8 + ((size_t)(b * H + h) * Nq + r0) * D;
#pragma unroll
  for (int i = 0; i < SEG; ++i) {
    const int s = lane + 32 * i;
    const int row = s / SEG, col = (s % SEG) * 8;
    float f[8];
    unpack_bf16x8(x[i], f);
    uint2 o;
    o.x = i8_code(f[0], inv) | i8_code(f[1], inv) << 8 | i8_code(f[2], inv) << 16 | i8_code(f[3], inv) << 24;
    o.y = i8_code(f[4], inv) | i8_code(f[5], inv) << 8 | i8_code(f[6], inv) << 16 | i8_code(f[7], inv) << 24;
    *reinterpret_cast<uint2*>(dst + (size_t)row * D + col) = o;
  }
}

// K: one 128-thread block per 64-row block; x' = fl32(x - k_mean[d]).  The
// raw BF16 chunks stay in registers between the amax pass and the code pass
// (x' is recomputed, the same single rounding), which keeps the block small
// enough for many blocks per SM.
template <int D>
__global__ void __launch_bounds__(128, 8) quant_k_kernel(const uint16_t* __restrict__ k, int64_t sb,
                                                         int64_t sn, int64_t sh, int N, int H, int Nk,
                                                         int T64, const float* __restrict__ k_mean,
                                                         int8_t* __restrict__ k8,
                                                         float* __restrict__ k_scale) {
  constexpr int SEG = D / 8;
  constexpr int PER = kKTile * SEG / 128;
  const int t = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int col = (threadIdx.x % SEG) * 8;
  uint4 xr[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int row = t * kKTile + (threadIdx.x + 128 * i) / SEG;
    xr[i] = row < N ? ldg16(k + b * sb + (int64_t)row * sn + h * sh + col) : make_uint4(0, 0, 0, 0);
  }
  float km[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) km[j] = __ldg(k_mean + (size_t)(b * H + h) * D + col + j);
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int row = t * kKTile + (threadIdx.x + 128 * i) / SEG;
    if (row < N) {
      float f[8];
      unpack_bf16x8(xr[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) amax = fmaxf(amax, fabsf(__fsub_rn(f[j], km[j])));
    }
  }
  __shared__ float red[4];
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  if (threadIdx.x == 0)
    k_scale[(size_t)(b * H + h) * T64 + t] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  int8_t* dst = k8 + ((size_t)(b * H + h) * Nk + (size_t)t * kKTile) * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int r = (threadIdx.x + 128 * i) / SEG;
    uint2 o = make_uint2(0u, 0u);  // pad rows get zero codes
    if (t * kKTile + r < N) {
      float f[8];
      unpack_bf16x8(xr[i], f);
      float x[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) x[j] = __fsub_rn(f[j], km[j]);
      o.x = i8_code(x[0], inv) | i8_code(x[1], inv) << 8 | i8_code(x[2], inv) << 16 | i8_code(x[3], inv) << 24;
      o.y = i8_code(x[4], inv) | i8_code(x[5], inv) << 8 | i8_code(x[6], inv) << 16 | i8_code(x[7], inv) << 24;
    }
    *reinterpret_cast<uint2*>(dst + (size_t)r * D + col) = o;
  }
}

// V: one 256-thread block per 128 tokens of one head.  The BF16 rows are
// staged in shared memory with 16-byte loads; the 16-byte chunk index of a
// row is XORed with bits 4-5 of its token, so that the column reads below
// (four 16-token runs x eight channels per warp) fall in distinct banks.
// Each thread then converts 16 consecutive tokens of one channel to E4M3
// (two tokens per conversion, the earlier token in the low byte, so token t
// is byte t of the channel's row) and writes them as one 16-byte vector; a
// warp writes eight channels x 64 contiguous bytes.
constexpr int kVTokens = 2 * kKTile;  // tokens per quant_v block

template <int D>
__global__ void __launch_bounds__(256) quant_v_kernel(const uint16_t* __restrict__ v, int64_t sb,
                                                      int64_t sn, int64_t sh, int N, int H, int Nk,
                                                      const float* __restrict__ v_amax,
                                                      uint8_t* __restrict__ v8) {
  constexpr int SEG = D / 8;                   // 16-byte chunks per token row
  constexpr int LOADS = kVTokens * SEG / 256;  // chunks staged per thread
  constexpr int RUNS = D * (kVTokens / 16) / 256;  // 16-token runs converted per thread
  __shared__ __align__(16) uint4 tile[kVTokens * SEG];
  const int h = blockIdx.y, b = blockIdx.z;
  const int n0 = blockIdx.x * kVTokens;
  const uint16_t* vp = v + b * sb + h * sh;
  uint4 x[LOADS];
#pragma unroll
  for (int i = 0; i < LOADS; ++i) {
    const int idx = threadIdx.x + 256 * i;
    const int r = idx / SEG, k = idx % SEG;
    x[i] = n0 + r < N ? ldg16(vp + (int64_t)(n0 + r) * sn + k * 8) : make_uint4(0, 0, 0, 0);
  }
#pragma unroll
  for (int i = 0; i < LOADS; ++i) {
    const int idx = threadIdx.x + 256 * i;
    const int r = idx / SEG, k = idx % SEG;
    tile[r * SEG + (k ^ ((r >> 4) & 3))] = x[i];
  }
  __syncthreads();
  const uint16_t* ts = reinterpret_cast<const uint16_t*>(tile);
  const float* am = v_amax + (size_t)(b * H + h) * D;
#pragma unroll
  for (int i = 0; i < RUNS; ++i) {
    const int idx = threadIdx.x + 256 * i;
    const int q = idx & 3, cl = (idx >> 2) & 7, rest = idx >> 5;
    const int cb = rest % SEG, half = rest / SEG;
    const int t0 = half * kKTile + 16 * q;  // first token of the run; (t >> 4) & 3 == q
    if (n0 + half * kKTile >= Nk) continue;  // past the padded length
    const int ch = cb * 8 + cl;
    const float a = am[ch];
    const float inv = a > 0.0f ? __fdiv_rn(448.0f, a) : 0.0f;
    const uint16_t* col = ts + (cb ^ q) * 8 + cl;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + 4 * j;
      const uint32_t lo = e4m3x2(__fmul_rn(bf16_bits_to_f32(col[t * D]), inv),
                                 __fmul_rn(bf16_bits_to_f32(col[(t + 1) * D]), inv));
      const uint32_t hi = e4m3x2(__fmul_rn(bf16_bits_to_f32(col[(t + 2) * D]), inv),
                                 __fmul_rn(bf16_bits_to_f32(col[(t + 3) * D]), inv));
      w[j] = a > 0.0f ? (lo | (hi << 16)) : 0u;
    }
    uint8_t* dst = v8 + ((size_t)(b * H + h) * D + ch) * Nk + n0 + t0;
    *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

int check_launch() { return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

template <int D>
int prepass_qk(const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H, int8_t* q8,
               float* q_scale, int8_t* k8, float* k_scale, float* k_mean, double* k_part,
               cudaStream_t s) {
  const int Nq = ceil_div(N, kQTile) * kQTile, T64 = ceil_div(N, kKTile), Nk = T64 * kKTile;
  const int G32 = ceil_div(N, kQGroup);
  const uint16_t* qp = static_cast<const uint16_t*>(q.data);
  const uint16_t* kp = static_cast<const uint16_t*>(k.data);
  constexpr int CPB = 128 / (D / 8);
  chunk_stats_kernel<D, true, false><<<dim3(ceil_div(T64, CPB), H, B), 128, 0, s>>>(
      kp, k.stride_b, k.stride_n, k.stride_h, nullptr, 0, 0, 0, N, H, T64, k_part, nullptr);
  reduce_stats_kernel<true, false><<<B * H, D, 0, s>>>(N, D, T64, k_part, k_mean, nullptr, nullptr,
                                                       nullptr);
  quant_q_kernel<D><<<dim3(Nq / kQTile, H, B), 128, 0, s>>>(qp, q.stride_b, q.stride_n, q.stride_h,
                                                            N, H, Nq, G32, q8, q_scale);
  quant_k_kernel<D><<<dim3(T64, H, B), 128, 0, s>>>(kp, k.stride_b, k.stride_n, k.stride_h, N, H,
                                                    Nk, T64, k_mean, k8, k_scale);
  return check_launch();
}

template <int D>
int prepass_v(const sage_view_bf16& v, int B, int N, int H, uint8_t* v8, float* v_scale,
              float* v_part, float* v_amax, cudaStream_t s) {
  const int T64 = ceil_div(N, kKTile), Nk = T64 * kKTile;
  const uint16_t* vp = static_cast<const uint16_t*>(v.data);
  constexpr int CPB = 128 / (D / 8);
  chunk_stats_kernel<D, false, true><<<dim3(ceil_div(T64, CPB), H, B), 128, 0, s>>>(
      nullptr, 0, 0, 0, vp, v.stride_b, v.stride_n, v.stride_h, N, H, T64, nullptr, v_part);
  reduce_stats_kernel<false, true><<<B * H, D, 0, s>>>(N, D, T64, nullptr, nullptr, v_part, v_scale,
                                                       v_amax);
  quant_v_kernel<D><<<dim3(ceil_div(Nk, kVTokens), H, B), 256, 0, s>>>(vp, v.stride_b, v.stride_n,
                                                                       v.stride_h, N, H, Nk, v_amax, v8);
  return check_launch();
}

}  // namespace

void launch_reduce_k_mean(int BH, int N, int D, int T64, const double* k_part, float* k_mean, cudaStream_t s) {
  reduce_stats_kernel<true, false><<<BH, D, 0, s>>>(N, D, T64, k_part, k_mean, nullptr, nullptr, nullptr);
}

int launch_prepass_qk(const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H, int D,
                      int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                      double* k_part, cudaStream_t s) {
  if (D == 128) return prepass_qk<128>(q, k, B, N, H, q8, q_scale, k8, k_scale, k_mean, k_part, s);
  if (D == 64) return prepass_qk<64>(q, k, B, N, H, q8, q_scale, k8, k_scale, k_mean, k_part, s);
  return SAGE_ERR_UNSUPPORTED;
}

int launch_prepass_v(const sage_view_bf16& v, int B, int N, int H, int D, uint8_t* v8,
                     float* v_scale, float* v_part, float* v_amax, cudaStream_t s) {
  if (D == 128) return prepass_v<128>(v, B, N, H, v8, v_scale, v_part, v_amax, s);
  if (D == 64) return prepass_v<64>(v, B, N, H, v8, v_scale, v_part, v_amax, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
