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
#include "prepass_codes.cuh"

namespace sage {
namespace {

__device__ __forceinline__ uint4 ldg16(const uint16_t* p) {
  return __ldg(reinterpret_cast<const uint4*>(p));
}

// ------------------------------------------------------------------------
// K: per 64-token chunk, the FP64 sum of each channel (tokens added in
// order).  One thread owns 8 consecutive channels of one chunk; D/8 threads
// per chunk; 128 threads per block.
template <int D>
__global__ void __launch_bounds__(128, 8) k_sums_kernel(const uint16_t* __restrict__ k, int64_t sb, int64_t sn,
                                                     int64_t sh, int N, int H, int T64,
                                                     double* __restrict__ k_part) {
  constexpr int TPC = D / 8;
  constexpr int CPB = 128 / TPC;
  const int chunk = blockIdx.x * CPB + threadIdx.x / TPC;
  const int col = (threadIdx.x % TPC) * 8;
  const int h = blockIdx.y, b = blockIdx.z;
  if (chunk >= T64) return;
  const int n0 = chunk * kKTile;
  const int n1 = min(n0 + kKTile, N);
  double ks[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) ks[i] = 0.0;
  const uint16_t* kp = k + b * sb + h * sh + col;
#pragma unroll 4
  for (int n = n0; n < n1; ++n) {
    float f[8];
    unpack_bf16x8(ldg16(kp + n * sn), f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ks[i] = __dadd_rn(ks[i], (double)f[i]);
  }
  double2* dst = reinterpret_cast<double2*>(k_part + (((size_t)b * H + h) * T64 + chunk) * D + col);
#pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = make_double2(ks[2 * i], ks[2 * i + 1]);
}

// Chunk partials -> k_mean: the partials added in chunk order, then one FP64
// division and one rounding to FP32.  One 128-thread block per head; pieces
// of kKMeanPiece chunks x D partials are copied into shared memory with
// cp.async (two buffers: the next piece streams in while thread d < D adds
// channel d of the current one), so the sequential sums run from shared
// memory instead of waiting on each load.
constexpr int kKMeanPiece = 32;

template <int D>
__global__ void __launch_bounds__(128) k_mean_kernel(int N, int T64, const double* __restrict__ k_part,
                                                     float* __restrict__ k_mean) {
  extern __shared__ __align__(16) double kbuf[];  // [2][kKMeanPiece][D]
  const size_t bh = blockIdx.x;
  const double* src = k_part + bh * T64 * D;
  const int pieces = ceil_div(T64, kKMeanPiece);
  auto fetch = [&](int pc) {
    const int c0 = pc * kKMeanPiece, n = min(kKMeanPiece, T64 - c0);
    double* dst = kbuf + (pc & 1) * kKMeanPiece * D;
    for (int i = threadIdx.x; i < n * D / 2; i += 128)  // 16-byte pairs of doubles
      cp_async_16(smem_u32(dst + 2 * i), src + (size_t)c0 * D + 2 * i);
    cp_async_commit();
  };
  fetch(0);
  double total = 0.0;
  for (int pc = 0; pc < pieces; ++pc) {
    if (pc + 1 < pieces) {
      fetch(pc + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    const int n = min(kKMeanPiece, T64 - pc * kKMeanPiece);
    const double* cur = kbuf + (pc & 1) * kKMeanPiece * D;
    if (threadIdx.x < D)
      for (int c = 0; c < n; ++c) total = __dadd_rn(total, cur[c * D + threadIdx.x]);
    __syncthreads();  // the buffer is refilled two pieces on
  }
  if (threadIdx.x < D) k_mean[bh * D + threadIdx.x] = __double2float_rn(__ddiv_rn(total, (double)N));
}

template <int D>
void launch_k_mean(int BH, int N, int T64, const double* k_part, float* k_mean, cudaStream_t s) {
  const size_t smem = 2 * kKMeanPiece * D * sizeof(double);  // 64 KB at D = 128
  cudaFuncSetAttribute(k_mean_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  k_mean_kernel<D><<<BH, 128, smem, s>>>(N, T64, k_part, k_mean);
}

// V: the FP32 amax of each channel over all tokens.  A block takes 8 * 128/D
// chunks of 64 tokens, reduces them in shared memory and merges the result
// into v_amax[b][h][d] (zero at the launch) with an integer atomic max: the
// amax of non-negative floats is exact in any order, and their bit patterns
// order as integers.
template <int D>
__global__ void __launch_bounds__(128) v_amax_kernel(const uint16_t* __restrict__ v, int64_t sb, int64_t sn,
                                                     int64_t sh, int N, int H, int T64, float* __restrict__ v_amax) {
  constexpr int TPC = D / 8;
  constexpr int CPB = 128 / TPC;
  __shared__ float red[CPB][D];
  const int cl = threadIdx.x / TPC;
  const int chunk = blockIdx.x * CPB + cl;
  const int col = (threadIdx.x % TPC) * 8;
  const int h = blockIdx.y, b = blockIdx.z;
  float vm[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) vm[i] = 0.0f;
  if (chunk < T64) {
    const int n0 = chunk * kKTile;
    const int n1 = min(n0 + kKTile, N);
    const uint16_t* vp = v + b * sb + h * sh + col;
#pragma unroll 4
    for (int n = n0; n < n1; ++n) {
      float f[8];
      unpack_bf16x8(ldg16(vp + n * sn), f);
#pragma unroll
      for (int i = 0; i < 8; ++i) vm[i] = fmaxf(vm[i], fabsf(f[i]));
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) red[cl][col + i] = vm[i];
  __syncthreads();
  if (threadIdx.x < D) {
    float am = red[0][threadIdx.x];
#pragma unroll
    for (int c = 1; c < CPB; ++c) am = fmaxf(am, red[c][threadIdx.x]);
    atomicMax(reinterpret_cast<int*>(v_amax) + ((size_t)b * H + h) * D + threadIdx.x, __float_as_int(am));
  }
}

// ------------------------------------------------------------------------
// Q: one 128-thread block per 64 rows (two 32-row groups, each with its own
// scale).  Thread t holds 16-byte segments t + 128 i of the 64 x D block in
// registers between the amax pass and the code pass; its first PER/2
// segments lie in group 0, the rest in group 1.  Pad rows get zero codes,
// pad groups no scale.
template <int D>
__global__ void __launch_bounds__(128, 6) quant_q_kernel(const uint16_t* __restrict__ q, int64_t sb,
                                                         int64_t sn, int64_t sh, int N, int H, int Nq,
                                                         int G32, int8_t* __restrict__ q8,
                                                         float* __restrict__ q_scale) {
  constexpr int SEG = D / 8;
  constexpr int PER = 2 * kQGroup * SEG / 128;  // segments per thread (8 at D = 128)
  const int blk = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int col = (threadIdx.x % SEG) * 8;
  const int r0 = blk * 2 * kQGroup;
  uint4 xr[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int row = r0 + (threadIdx.x + 128 * i) / SEG;
    xr[i] = row < N ? ldg16(q + b * sb + (int64_t)row * sn + h * sh + col) : make_uint4(0, 0, 0, 0);
  }
  // amax as BF16 magnitude bits (NaN and inf above every finite value)
  uint32_t mb[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < PER; ++i) mb[i / (PER / 2)] = amax_bits8(xr[i], mb[i / (PER / 2)]);
  __shared__ uint32_t redb[2][4];
  __shared__ float red[2][4];
#pragma unroll
  for (int g = 0; g < 2; ++g) mb[g] = __reduce_max_sync(0xffffffffu, halves_max(mb[g]));
  if ((threadIdx.x & 31) == 0) {
    redb[0][threadIdx.x >> 5] = mb[0];
    redb[1][threadIdx.x >> 5] = mb[1];
  }
  __syncthreads();
  float a[2];
  bool finite[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    mb[g] = max(max(redb[g][0], redb[g][1]), max(redb[g][2], redb[g][3]));
    finite[g] = mb[g] < 0x7F80u;
    a[g] = __uint_as_float(mb[g] << 16);
  }
  if (!finite[0] || !finite[1]) {
    // NaN or inf in the block: the amax that ignores NaN (the reference form)
    float am[2] = {0.0f, 0.0f};
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      float f[8];
      unpack_bf16x8(xr[i], f);
#pragma unroll
      for (int j = 0; j < 8; ++j) am[i / (PER / 2)] = fmaxf(am[i / (PER / 2)], fabsf(f[j]));
    }
    am[0] = warp_max(am[0]);
    am[1] = warp_max(am[1]);
    if ((threadIdx.x & 31) == 0) {
      red[0][threadIdx.x >> 5] = am[0];
      red[1][threadIdx.x >> 5] = am[1];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < 2; ++g) a[g] = fmaxf(fmaxf(red[g][0], red[g][1]), fmaxf(red[g][2], red[g][3]));
  }
  float inv[2];
  bool fast[2];
#pragma unroll
  for (int g = 0; g < 2; ++g) {
    inv[g] = a[g] > 0.0f ? __fdiv_rn(127.0f, a[g]) : 0.0f;
    fast[g] = finite[g] && codes_fast(a[g], inv[g]);
    const int grp = 2 * blk + g;
    if (threadIdx.x == 0 && grp < G32)
      q_scale[(size_t)(b * H + h) * G32 + grp] = a[g] > 0.0f ? __fdiv_rn(a[g], 127.0f) : 0.0f;
  }
  int8_t* dst = q8 + ((size_t)(b * H + h) * Nq + r0) * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int r = (threadIdx.x + 128 * i) / SEG;
    const float iv = inv[i / (PER / 2)];
    float f[8];
    unpack_bf16x8(xr[i], f);  // pad rows were loaded as zeros: zero codes
    const uint2 o = fast[i / (PER / 2)] ? i8_codes8_fast(f, iv) : i8_codes8_ref(f, iv);
    *reinterpret_cast<uint2*>(dst + (size_t)r * D + col) = o;
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
  // heads in the reverse of the statistics pass's order: the K rows it read
  // last are still in L2
  const int t = blockIdx.x, h = H - 1 - (int)blockIdx.y, b = (int)gridDim.z - 1 - (int)blockIdx.z;
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
      for (int j = 0; j < 8; ++j) amax = fmax_nan(amax, fabsf(__fsub_rn(f[j], km[j])));
    }
  }
  // the bits of non-negative floats order as integers, NaN above inf
  __shared__ uint32_t redb[4];
  __shared__ float red[4];
  uint32_t ab = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));
  if ((threadIdx.x & 31) == 0) redb[threadIdx.x >> 5] = ab;
  __syncthreads();
  ab = max(max(redb[0], redb[1]), max(redb[2], redb[3]));
  const bool finite = ab < 0x7F800000u;
  amax = __uint_as_float(ab);
  if (!finite) {
    // NaN or inf in the block: the amax that ignores NaN (the reference form)
    amax = 0.0f;
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
    amax = warp_max(amax);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
    __syncthreads();
    amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  }
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  const bool fast = finite && codes_fast(amax, inv);
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
      o = fast ? i8_codes8_fast(x, inv) : i8_codes8_ref(x, inv);
    }
    *reinterpret_cast<uint2*>(dst + (size_t)r * D + col) = o;
  }
}

// V: one 256-thread block per 128 tokens of one head.  The BF16 rows are
// copied into shared memory with cp.async (rows past N zero-filled); the
// 16-byte piece k of row r is stored at k ^ (2 * ((r >> 4) & 3)).  Each
// thread then takes two adjacent channels of 16 consecutive tokens: one
// 4-byte shared load per token gives both channels, and the loads of a warp
// (four 16-token runs x eight channel pairs over two pieces) fall in 32
// distinct banks.  Each channel's 16 tokens are converted to E4M3 (two
// tokens per conversion, the earlier token in the low byte, so token t is
// byte t of the channel's row) and written as one 16-byte vector; a warp
// writes 16 channels x 64 contiguous bytes.
constexpr int kVTokens = 2 * kKTile;  // tokens per quant_v block

template <int D>
__global__ void __launch_bounds__(256) quant_v_kernel(const uint16_t* __restrict__ v, int64_t sb,
                                                      int64_t sn, int64_t sh, int N, int H, int Nk,
                                                      const float* __restrict__ v_amax,
                                                      uint8_t* __restrict__ v8, float* __restrict__ v_scale) {
  constexpr int SEG = D / 8;                          // 16-byte pieces per token row
  constexpr int COPIES = kVTokens * SEG / 256;        // pieces copied per thread
  constexpr int RUNS = (D / 2) * (kVTokens / 16) / 256;  // (channel pair, 16-token run)s per thread
  __shared__ __align__(16) uint4 tile[kVTokens * SEG];
  // the last prepass kernel: the mainloop that follows may start its set-up
  // (it waits for this grid to complete before it reads anything written here)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // heads in the reverse of the statistics pass's order (its last rows are
  // still in L2)
  const int h = H - 1 - (int)blockIdx.y, b = (int)gridDim.z - 1 - (int)blockIdx.z;
  const int n0 = blockIdx.x * kVTokens;
  const uint16_t* vp = v + b * sb + h * sh;
  const uint32_t ts0 = smem_u32(tile);
#pragma unroll
  for (int i = 0; i < COPIES; ++i) {
    const int idx = threadIdx.x + 256 * i;
    const int r = idx / SEG, k = idx % SEG;
    const bool valid = n0 + r < N;
    cp_async_16_zfill(ts0 + (uint32_t)((r * SEG + (k ^ (2 * ((r >> 4) & 3)))) * 16),
                      valid ? vp + (int64_t)(n0 + r) * sn + k * 8 : vp, valid);
  }
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  const uint8_t* tb = reinterpret_cast<const uint8_t*>(tile);
  const float* am = v_amax + (size_t)(b * H + h) * D;
#pragma unroll
  for (int i = 0; i < RUNS; ++i) {
    const int idx = threadIdx.x + 256 * i;
    const int q = idx & 3, cp = (idx >> 2) & 7, rest = idx >> 5;
    const int pg = rest % (SEG / 2), half = rest / (SEG / 2);
    const int t0 = half * kKTile + 16 * q;  // first token of the run; (t >> 4) & 3 == q
    if (n0 + half * kKTile >= Nk) continue;  // past the padded length
    const int c0 = pg * 16 + 2 * cp;        // channels c0, c0 + 1
    const int k = c0 >> 3;                  // their piece
    const float a0 = am[c0], a1 = am[c0 + 1];
    const float i0 = a0 > 0.0f ? __fdiv_rn(448.0f, a0) : 0.0f;
    const float i1 = a1 > 0.0f ? __fdiv_rn(448.0f, a1) : 0.0f;
    if (n0 == 0 && t0 == 0) {  // the channels' scales, once per head
      v_scale[(size_t)(b * H + h) * D + c0] = a0 > 0.0f ? __fdiv_rn(a0, 448.0f) : 0.0f;
      v_scale[(size_t)(b * H + h) * D + c0 + 1] = a1 > 0.0f ? __fdiv_rn(a1, 448.0f) : 0.0f;
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
    uint8_t* dst = v8 + ((size_t)(b * H + h) * D + c0) * Nk + n0 + t0;
    *reinterpret_cast<uint4*>(dst) = make_uint4(wa[0], wa[1], wa[2], wa[3]);
    *reinterpret_cast<uint4*>(dst + Nk) = make_uint4(wc[0], wc[1], wc[2], wc[3]);
  }
}

int check_launch() { return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA; }

template <int D>
int prepass_qk(const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H, int8_t* q8,
               float* q_scale, int8_t* k8, float* k_scale, float* k_mean, double* k_part, cudaStream_t s) {
  const int Nq = ceil_div(N, kQTile) * kQTile, T64 = ceil_div(N, kKTile), Nk = T64 * kKTile;
  const int G32 = ceil_div(N, kQGroup);
  const uint16_t* qp = static_cast<const uint16_t*>(q.data);
  const uint16_t* kp = static_cast<const uint16_t*>(k.data);
  constexpr int CPB = 128 / (D / 8);
  k_sums_kernel<D><<<dim3(ceil_div(T64, CPB), H, B), 128, 0, s>>>(kp, k.stride_b, k.stride_n, k.stride_h, N, H,
                                                                  T64, k_part);
  launch_k_mean<D>(B * H, N, T64, k_part, k_mean, s);
  // K right after its statistics (part of K is still in L2), then Q
  quant_k_kernel<D><<<dim3(T64, H, B), 128, 0, s>>>(kp, k.stride_b, k.stride_n, k.stride_h, N, H,
                                                    Nk, T64, k_mean, k8, k_scale);
  quant_q_kernel<D><<<dim3(Nq / (2 * kQGroup), H, B), 128, 0, s>>>(qp, q.stride_b, q.stride_n, q.stride_h,
                                                                   N, H, Nq, G32, q8, q_scale);
  return check_launch();
}

template <int D>
int prepass_v(const sage_view_bf16& v, int B, int N, int H, uint8_t* v8, float* v_scale, float* v_amax,
              cudaStream_t s) {
  const int T64 = ceil_div(N, kKTile), Nk = T64 * kKTile;
  const uint16_t* vp = static_cast<const uint16_t*>(v.data);
  constexpr int CPB = 128 / (D / 8);
  if (cudaMemsetAsync(v_amax, 0, sizeof(float) * (size_t)B * H * D, s) != cudaSuccess) return SAGE_ERR_CUDA;
  v_amax_kernel<D><<<dim3(ceil_div(T64, CPB), H, B), 128, 0, s>>>(vp, v.stride_b, v.stride_n, v.stride_h, N, H,
                                                                  T64, v_amax);
  quant_v_kernel<D><<<dim3(ceil_div(Nk, kVTokens), H, B), 256, 0, s>>>(vp, v.stride_b, v.stride_n,
                                                                       v.stride_h, N, H, Nk, v_amax, v8, v_scale);
  return check_launch();
}

}  // namespace

void launch_reduce_k_mean(int BH, int N, int D, int T64, const double* k_part, float* k_mean, cudaStream_t s) {
  if (D == 128) launch_k_mean<128>(BH, N, T64, k_part, k_mean, s);
  else if (D == 64) launch_k_mean<64>(BH, N, T64, k_part, k_mean, s);
}

int launch_prepass_qk(const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H, int D,
                      int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                      double* k_part, cudaStream_t s) {
  if (D == 128) return prepass_qk<128>(q, k, B, N, H, q8, q_scale, k8, k_scale, k_mean, k_part, s);
  if (D == 64) return prepass_qk<64>(q, k, B, N, H, q8, q_scale, k8, k_scale, k_mean, k_part, s);
  return SAGE_ERR_UNSUPPORTED;
}

int launch_prepass_v(const sage_view_bf16& v, int B, int N, int H, int D, uint8_t* v8,
                     float* v_scale, float* v_amax, cudaStream_t s) {
  if (D == 128) return prepass_v<128>(v, B, N, H, v8, v_scale, v_amax, s);
  if (D == 64) return prepass_v<64>(v, B, N, H, v8, v_scale, v_amax, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
