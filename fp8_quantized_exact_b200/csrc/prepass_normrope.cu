// Q/K producer with RMSNorm and split-half RoPE in front of the INT8
// quantisation: one thread per (b, n, h) row normalises and rotates it in
// registers, then the row goes through the same Q/K rules as the raw
// producer (K channel mean in FP64, K smoothing, per-32-row INT8 Q,
// per-64-row INT8 K).  The normalised rows are never written to memory; the
// K quantisation recomputes them.
//
// Operation: the fused strided-NHD Q/K RMSNorm + split-half RoPE + INT8
// producer of "Sage2 Blackwell Mainloop", section "Completed P1 And P2".
// The pages give no formula or rounding; the reading used, per row x of D
// BF16 values with BF16 weight w and FP32 tables cos/sin[N][D/2]:
//   ss = FP32 sum of fl32(x_d * x_d) in channel order;
//   r  = fl32(1 / fl32(sqrt(fl32(fl32(ss / D) + eps))))  (correctly rounded);
//   y_d = bf16(fl32(bf16(fl32(x_d * r)) * w_d));
//   z_j = bf16(fl32(fl32(y_j c) - fl32(y_{j+D/2} s))),
//   z_{j+D/2} = bf16(fl32(fl32(y_{j+D/2} c) + fl32(y_j s))),  c, s = cos/sin[n][j].
#include "sage_common.cuh"

namespace sage {
namespace {

__device__ __forceinline__ float lo_bf16(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float hi_bf16(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// The row (D BF16 values, 16-byte aligned) normalised and rotated; z holds
// D/2 words of two BF16 values each (channel 2i in the low half).
template <int D>
__device__ __forceinline__ void norm_rope_row(const uint16_t* row, const uint16_t* __restrict__ w,
                                              const float* __restrict__ cs, const float* __restrict__ sn,
                                              float eps, uint32_t (&z)[D / 2]) {
  constexpr int HALF = D / 2;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + i);
    z[4 * i] = u.x; z[4 * i + 1] = u.y; z[4 * i + 2] = u.z; z[4 * i + 3] = u.w;
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const float a = lo_bf16(z[i]), b = hi_bf16(z[i]);
    ss = __fadd_rn(ss, __fmul_rn(a, a));
    ss = __fadd_rn(ss, __fmul_rn(b, b));
  }
  const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(ss, (float)D), eps)));
  // y = bf16(bf16(x * r) * w), in place
#pragma unroll
  for (int i = 0; i < HALF; ++i) {
    const uint32_t ww = __ldg(reinterpret_cast<const uint32_t*>(w) + i);
    const float y0 = __fmul_rn(bf16_bits_to_f32(f32_to_bf16_rn(__fmul_rn(lo_bf16(z[i]), r))), lo_bf16(ww));
    const float y1 = __fmul_rn(bf16_bits_to_f32(f32_to_bf16_rn(__fmul_rn(hi_bf16(z[i]), r))), hi_bf16(ww));
    z[i] = (uint32_t)f32_to_bf16_rn(y0) | ((uint32_t)f32_to_bf16_rn(y1) << 16);
  }
  // rotate channel j with channel j + D/2 (words i and i + D/4 hold them)
#pragma unroll
  for (int i = 0; i < D / 4; ++i) {
    const uint32_t wa = z[i], wb = z[i + D / 4];
    const float2 c = __ldg(reinterpret_cast<const float2*>(cs) + i);
    const float2 s = __ldg(reinterpret_cast<const float2*>(sn) + i);
    const float a0 = lo_bf16(wa), a1 = hi_bf16(wa), b0 = lo_bf16(wb), b1 = hi_bf16(wb);
    const uint32_t z0 = f32_to_bf16_rn(__fsub_rn(__fmul_rn(a0, c.x), __fmul_rn(b0, s.x)));
    const uint32_t z1 = f32_to_bf16_rn(__fsub_rn(__fmul_rn(a1, c.y), __fmul_rn(b1, s.y)));
    const uint32_t z2 = f32_to_bf16_rn(__fadd_rn(__fmul_rn(b0, c.x), __fmul_rn(a0, s.x)));
    const uint32_t z3 = f32_to_bf16_rn(__fadd_rn(__fmul_rn(b1, c.y), __fmul_rn(a1, s.y)));
    z[i] = z0 | (z1 << 16);
    z[i + D / 4] = z2 | (z3 << 16);
  }
}

__device__ __forceinline__ uint32_t code8(float x, float inv) {
  int r = __float2int_rn(__fmul_rn(x, inv));
  r = max(-127, min(127, r));
  return static_cast<uint32_t>(r) & 0xFFu;
}

struct NormRopeArgs {
  const uint16_t* x;
  int64_t sb, sn, sh;
  const uint16_t* w;
  const float* cos_t;
  const float* sin_t;
  float eps;
  int B, N, H;
};

// Q: one thread per row, one warp per 32-row group; pad rows are zeros.
template <int D>
__global__ void __launch_bounds__(128) nr_quant_q_kernel(const NormRopeArgs a, int Nq, int G32, int8_t* __restrict__ q8,
                                                         float* __restrict__ q_scale) {
  const int h = blockIdx.y, b = blockIdx.z;
  const int row = blockIdx.x * kQTile + threadIdx.x;
  uint32_t z[D / 2];
  if (row < a.N) {
    norm_rope_row<D>(a.x + b * a.sb + (int64_t)row * a.sn + h * a.sh, a.w, a.cos_t + (size_t)row * (D / 2),
                     a.sin_t + (size_t)row * (D / 2), a.eps, z);
  } else {
#pragma unroll
    for (int i = 0; i < D / 2; ++i) z[i] = 0u;
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < D / 2; ++i) amax = fmaxf(amax, fmaxf(fabsf(lo_bf16(z[i])), fabsf(hi_bf16(z[i]))));
  amax = warp_max(amax);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  const int g = row / kQGroup;
  if ((threadIdx.x & 31) == 0 && g < G32)
    q_scale[(size_t)(b * a.H + h) * G32 + g] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  int8_t* dst = q8 + ((size_t)(b * a.H + h) * Nq + row) * D;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    uint32_t o[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t w0 = z[4 * i + 2 * k], w1 = z[4 * i + 2 * k + 1];
      o[k] = code8(lo_bf16(w0), inv) | code8(hi_bf16(w0), inv) << 8 | code8(lo_bf16(w1), inv) << 16 |
             code8(hi_bf16(w1), inv) << 24;
    }
    *reinterpret_cast<uint2*>(dst + 8 * i) = make_uint2(o[0], o[1]);
  }
}

// K statistics: one 64-thread block per 64-token chunk; the normalised rows
// go through shared memory, then one thread per channel adds them in token
// order in FP64 (the same partials as the raw producer's chunk sums).
template <int D>
__global__ void __launch_bounds__(64) nr_kstats_kernel(const NormRopeArgs a, int T64, double* __restrict__ k_part) {
  __shared__ uint32_t zs[kKTile][D / 2];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int row = c * kKTile + threadIdx.x;
  uint32_t z[D / 2];
  if (row < a.N) {
    norm_rope_row<D>(a.x + b * a.sb + (int64_t)row * a.sn + h * a.sh, a.w, a.cos_t + (size_t)row * (D / 2),
                     a.sin_t + (size_t)row * (D / 2), a.eps, z);
  } else {
#pragma unroll
    for (int i = 0; i < D / 2; ++i) z[i] = 0u;
  }
#pragma unroll
  for (int i = 0; i < D / 2; ++i) zs[threadIdx.x][(i + threadIdx.x) % (D / 2)] = z[i];  // rotated: fewer bank conflicts
  __syncthreads();
  const int n1 = min(kKTile, a.N - c * kKTile);
  for (int d = threadIdx.x; d < D; d += kKTile) {
    const int wi = d >> 1;
    double s = 0.0;
    for (int t = 0; t < n1; ++t) {
      const uint32_t word = zs[t][(wi + t) % (D / 2)];
      s = __dadd_rn(s, (double)((d & 1) ? hi_bf16(word) : lo_bf16(word)));
    }
    k_part[((size_t)(b * a.H + h) * T64 + c) * D + d] = s;
  }
}

// K quantisation: one 64-thread block per 64-row block; x' = fl32(z - km).
template <int D>
__global__ void __launch_bounds__(64) nr_quant_k_kernel(const NormRopeArgs a, int Nk, int T64,
                                                        const float* __restrict__ k_mean, int8_t* __restrict__ k8,
                                                        float* __restrict__ k_scale) {
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int row = c * kKTile + threadIdx.x;
  const float* km = k_mean + (size_t)(b * a.H + h) * D;
  uint32_t z[D / 2];
  float amax = 0.0f;
  if (row < a.N) {
    norm_rope_row<D>(a.x + b * a.sb + (int64_t)row * a.sn + h * a.sh, a.w, a.cos_t + (size_t)row * (D / 2),
                     a.sin_t + (size_t)row * (D / 2), a.eps, z);
#pragma unroll
    for (int i = 0; i < D / 2; ++i) {
      const float x0 = __fsub_rn(lo_bf16(z[i]), __ldg(km + 2 * i));
      const float x1 = __fsub_rn(hi_bf16(z[i]), __ldg(km + 2 * i + 1));
      amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
    }
  }
  __shared__ float red[2];
  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(red[0], red[1]);
  const float inv = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  if (threadIdx.x == 0) k_scale[(size_t)(b * a.H + h) * T64 + c] = amax > 0.0f ? __fdiv_rn(amax, 127.0f) : 0.0f;
  int8_t* dst = k8 + ((size_t)(b * a.H + h) * Nk + row) * D;
#pragma unroll
  for (int i = 0; i < D / 8; ++i) {
    uint32_t o[2] = {0u, 0u};
    if (row < a.N) {
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int d = 8 * i + 4 * k;
        const uint32_t w0 = z[d / 2], w1 = z[d / 2 + 1];
        o[k] = code8(__fsub_rn(lo_bf16(w0), __ldg(km + d)), inv) |
               code8(__fsub_rn(hi_bf16(w0), __ldg(km + d + 1)), inv) << 8 |
               code8(__fsub_rn(lo_bf16(w1), __ldg(km + d + 2)), inv) << 16 |
               code8(__fsub_rn(hi_bf16(w1), __ldg(km + d + 3)), inv) << 24;
      }
    }
    *reinterpret_cast<uint2*>(dst + 8 * i) = make_uint2(o[0], o[1]);
  }
}

template <int D>
int run(const NormRopeIn& in, const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H, int8_t* q8,
        float* q_scale, int8_t* k8, float* k_scale, float* k_mean, double* k_part, cudaStream_t s) {
  const int Nq = ceil_div(N, kQTile) * kQTile, T64 = ceil_div(N, kKTile), Nk = T64 * kKTile;
  const int G32 = ceil_div(N, kQGroup);
  NormRopeArgs aq{static_cast<const uint16_t*>(q.data), q.stride_b, q.stride_n, q.stride_h, in.wq, in.cos_t,
                  in.sin_t, in.eps, B, N, H};
  NormRopeArgs ak{static_cast<const uint16_t*>(k.data), k.stride_b, k.stride_n, k.stride_h, in.wk, in.cos_t,
                  in.sin_t, in.eps, B, N, H};
  nr_quant_q_kernel<D><<<dim3(Nq / kQTile, H, B), 128, 0, s>>>(aq, Nq, G32, q8, q_scale);
  nr_kstats_kernel<D><<<dim3(T64, H, B), 64, 0, s>>>(ak, T64, k_part);
  launch_reduce_k_mean(B * H, N, D, T64, k_part, k_mean, s);
  nr_quant_k_kernel<D><<<dim3(T64, H, B), 64, 0, s>>>(ak, Nk, T64, k_mean, k8, k_scale);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

int launch_norm_rope_qk(const NormRopeIn& in, const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H,
                        int D, int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean, double* k_part,
                        cudaStream_t s) {
  if (D == 128) return run<128>(in, q, k, B, N, H, q8, q_scale, k8, k_scale, k_mean, k_part, s);
  if (D == 64) return run<64>(in, q, k, B, N, H, q8, q_scale, k8, k_scale, k_mean, k_part, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
