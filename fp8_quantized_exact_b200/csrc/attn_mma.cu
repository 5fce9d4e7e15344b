// Fused attention mainloop on warp-level mma.sync (the legacy tensor path).
//
// One CTA = one 128-row query tile of one (b, h); eight warps own 16 rows
// each.  K and V^T tiles of 64 keys are double-buffered in shared memory by
// cp.async.  Per tile and warp: INT8 m16n8k32 MMAs give the int32 scores,
// then the FP32 scale, the online-softmax max/denominator update, E4M3 P in
// registers, and per K32 slice one E4M3 m16n8k32 MMA with an FP16 accumulator
// that starts at zero, widened and added to the FP32 output accumulator.
//
// Operation: "State-Ownership Architecture Decision", section "Non-Negotiable
// Dataflow" (tile order, per-tile steps, two K32 FP16 PV MMAs then the FP32
// RO addition) and the exact handoff record (ro_rescale before the tile's
// PV; final FP32 reciprocal, then V scale, then BF16); per-tile step order
// from "Sage2 SM89 Temporal Pair Experiment", section "Candidate".
//
// Register layout trick: the QK^T B operand rows are gathered through
// ldmatrix row addresses so that each thread's int32 accumulators already
// sit in the positions of the PV A operand (no shuffles).  The n8 QK tile j
// holds, in its column n, the key
//   sigma(j, n) = 32*(j/4) + 16*((j%4)/2) + 4*(n/2) + 2*(j%2) + (n%2).
#include "sage_common.cuh"

namespace sage {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

__device__ __forceinline__ int key_of(int j, int n) {
  return 32 * (j >> 2) + 16 * ((j & 3) >> 1) + 4 * (n >> 1) + 2 * (j & 1) + (n & 1);
}

__device__ __forceinline__ void mma_s8(int32_t (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                       uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D(f16x2 x2) = A(e4m3) * B(e4m3) + 0
__device__ __forceinline__ void mma_e4m3_f16(uint32_t (&d)[2], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  const uint32_t z = 0u;
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f16.e4m3.e4m3.f16 {%0,%1}, {%2,%3,%4,%5}, {%6,%7}, "
      "{%8,%8};"
      : "=r"(d[0]), "=r"(d[1])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "r"(z));
}

// FP16 -> FP32 widening (exact) of the low / high half of an f16x2 word.
__device__ __forceinline__ float half_lo(uint32_t h2) {
  float f;
  asm("{.reg .b16 lo, hi; mov.b32 {lo, hi}, %1; cvt.f32.f16 %0, lo;}" : "=f"(f) : "r"(h2));
  return f;
}
__device__ __forceinline__ float half_hi(uint32_t h2) {
  float f;
  asm("{.reg .b16 lo, hi; mov.b32 {lo, hi}, %1; cvt.f32.f16 %0, hi;}" : "=f"(f) : "r"(h2));
  return f;
}

template <int D>
struct Smem {
  alignas(1024) uint8_t k[2][kKTile * D];  // [key][d], 128B-swizzled rows
  alignas(1024) uint8_t v[2][D * kKTile];  // [d][key], 128B-swizzled rows
};

// Stage the K tile (rows of D bytes) and the V^T tile (D rows of 64 bytes)
// of key tile t.  The quantised buffers are padded to Nk and the pads hold
// zeros, so no tile reads past its buffer.
template <int D>
__device__ __forceinline__ void load_k(Smem<D>& sm, int stage, const int8_t* kbase, int t) {
  constexpr int KCH = kKTile * D / 16;  // 16B chunks of the K tile
  const uint32_t ks = smem_u32(sm.k[stage]);
  const int8_t* ksrc = kbase + (size_t)t * kKTile * D;
  for (int i = threadIdx.x; i < KCH; i += kThreads) {
    const uint32_t off = i * 16u;  // row = off / D
    cp_async_16(ks + swz128(off), ksrc + off);
  }
}

template <int D>
__device__ __forceinline__ void load_v(Smem<D>& sm, int stage, const uint8_t* vbase, int Nk, int t) {
  constexpr int VCH = D * kKTile / 16;
  const uint32_t vs = smem_u32(sm.v[stage]);
  for (int i = threadIdx.x; i < VCH; i += kThreads) {
    const int d = i / (kKTile / 16), part = i % (kKTile / 16);
    const uint32_t off = d * kKTile + part * 16;
    cp_async_16(vs + swz128(off), vbase + (size_t)d * Nk + (size_t)t * kKTile + part * 16);
  }
}

template <int D>
__device__ __forceinline__ void load_tile(Smem<D>& sm, int stage, const int8_t* kbase,
                                          const uint8_t* vbase, int Nk, int t) {
  load_k<D>(sm, stage, kbase, t);
  load_v<D>(sm, stage, vbase, Nk, t);
}

// int32 scores of this warp's 16 rows against one staged K tile.
template <int D>
__device__ __forceinline__ void qk_tile(const Smem<D>& sm, int stage, const uint32_t (&qa)[D / 32][4],
                                        int32_t (&S)[8][4]) {
  const int lane = threadIdx.x & 31;
  const uint32_t kb = smem_u32(sm.k[stage]);
#pragma unroll
  for (int j = 0; j < 8; ++j) {
#pragma unroll
    for (int r = 0; r < 4; ++r) S[j][r] = 0;
    const int key = key_of(j, lane & 7);
#pragma unroll
    for (int ks = 0; ks < D / 32; ks += 2) {
      // matrices: (ks, k 0-15), (ks, k 16-31), (ks+1, k 0-15), (ks+1, k 16-31)
      const uint32_t off = key * D + (ks + (lane >> 4)) * 32 + ((lane >> 3) & 1) * 16;
      uint32_t b0, b1, b2, b3;
      ldmatrix_x4(kb + swz128(off), b0, b1, b2, b3);
      mma_s8(S[j], qa[ks], b0, b1);
      mma_s8(S[j], qa[ks + 1], b2, b3);
    }
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_mma_kernel(const AttnParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const size_t bh = (size_t)b * p.H + h;
  const int8_t* kbase = p.k8 + bh * p.Nk * D;
  const uint8_t* vbase = p.v8 + bh * D * p.Nk;
  const int T = p.T64;

  load_tile<D>(sm, 0, kbase, vbase, p.Nk, 0);
  cp_async_commit();

  // Q fragments of the warp's 16 rows, all of D.
  const int row0 = qt * kQTile + warp * 16;
  uint32_t qa[D / 32][4];
  {
    const int8_t* q0 = p.q8 + (bh * p.Nq + row0 + g) * D;
    const int8_t* q1 = q0 + 8 * D;
#pragma unroll
    for (int ks = 0; ks < D / 32; ++ks) {
      qa[ks][0] = __ldg(reinterpret_cast<const uint32_t*>(q0 + ks * 32 + 4 * c));
      qa[ks][1] = __ldg(reinterpret_cast<const uint32_t*>(q1 + ks * 32 + 4 * c));
      qa[ks][2] = __ldg(reinterpret_cast<const uint32_t*>(q0 + ks * 32 + 16 + 4 * c));
      qa[ks][3] = __ldg(reinterpret_cast<const uint32_t*>(q1 + ks * 32 + 16 + 4 * c));
    }
  }
  const int grp = row0 / kQGroup;
  const float qs = grp < p.G32 ? p.q_scale[bh * p.G32 + grp] : 0.0f;

  float RO[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int r = 0; r < 4; ++r) RO[i][r] = 0.0f;
  float m0 = -INFINITY, m1 = -INFINITY;  // rows g and g+8
  float d0 = 0.0f, d1 = 0.0f;            // this lane's share of the denominators

  for (int t = 0; t < T; ++t) {
    if (t + 1 < T) load_tile<D>(sm, (t + 1) & 1, kbase, vbase, p.Nk, t + 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const int st = t & 1;

    int32_t S[8][4];
    qk_tile<D>(sm, st, qa, S);

    // score scale for (Q32 group, K64 tile); masked keys beyond N
    const float cs = __fmul_rn(__fmul_rn(qs, p.k_scale[bh * T + t]), p.sl2);
    float s[8][4];
    float t0 = -INFINITY, t1 = -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int key = t * kKTile + key_of(j, 2 * c + (r & 1));
        const float v = key < p.N ? __fmul_rn(__int2float_rn(S[j][r]), cs) : -INFINITY;
        s[j][r] = v;
      }
      t0 = fmaxf(t0, fmaxf(s[j][0], s[j][1]));
      t1 = fmaxf(t1, fmaxf(s[j][2], s[j][3]));
    }
    t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, 1));
    t0 = fmaxf(t0, __shfl_xor_sync(0xffffffffu, t0, 2));
    t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, 1));
    t1 = fmaxf(t1, __shfl_xor_sync(0xffffffffu, t1, 2));
    const float mn0 = fmaxf(m0, t0), mn1 = fmaxf(m1, t1);
    const float r0 = mn0 == m0 ? 1.0f : exp2f(__fsub_rn(m0, mn0));
    const float r1 = mn1 == m1 ? 1.0f : exp2f(__fsub_rn(m1, mn1));
    m0 = mn0;
    m1 = mn1;
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      RO[i][0] = __fmul_rn(RO[i][0], r0);
      RO[i][1] = __fmul_rn(RO[i][1], r0);
      RO[i][2] = __fmul_rn(RO[i][2], r1);
      RO[i][3] = __fmul_rn(RO[i][3], r1);
    }
    d0 = __fmul_rn(d0, r0);
    d1 = __fmul_rn(d1, r1);

    // probabilities (FP32 into d), then E4M3 packed as the PV A operand
    uint32_t pa[2][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int r = 0; r < 4; ++r) s[j][r] = exp2f(__fsub_rn(s[j][r], (r < 2) ? m0 : m1));
      d0 = __fadd_rn(d0, __fadd_rn(s[j][0], s[j][1]));
      d1 = __fadd_rn(d1, __fadd_rn(s[j][2], s[j][3]));
    }
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        const int j0 = 4 * sl + 2 * half, j1 = j0 + 1;
        // row g: keys (j0, cols 2c, 2c+1), (j1, cols 2c, 2c+1)
        pa[sl][2 * half + 0] = (uint32_t)e4m3x2(s[j0][0], s[j0][1]) |
                               ((uint32_t)e4m3x2(s[j1][0], s[j1][1]) << 16);
        pa[sl][2 * half + 1] = (uint32_t)e4m3x2(s[j0][2], s[j0][3]) |
                               ((uint32_t)e4m3x2(s[j1][2], s[j1][3]) << 16);
      }
    }

    // PV: per K32 slice one FP16 instantaneous buffer, added into FP32 RO
    const uint32_t vb = smem_u32(sm.v[st]);
#pragma unroll
    for (int sl = 0; sl < 2; ++sl) {
#pragma unroll
      for (int nd = 0; nd < D / 8; nd += 2) {
        // matrices: (nd, keys 0-15), (nd, keys 16-31), (nd+1, 0-15), (nd+1, 16-31)
        const int drow = (nd + (lane >> 4)) * 8 + (lane & 7);
        const uint32_t off = drow * kKTile + sl * 32 + ((lane >> 3) & 1) * 16;
        uint32_t b0, b1, b2, b3;
        ldmatrix_x4(vb + swz128(off), b0, b1, b2, b3);
        uint32_t o0[2], o1[2];
        mma_e4m3_f16(o0, pa[sl], b0, b1);
        mma_e4m3_f16(o1, pa[sl], b2, b3);
        RO[nd][0] = __fadd_rn(RO[nd][0], half_lo(o0[0]));
        RO[nd][1] = __fadd_rn(RO[nd][1], half_hi(o0[0]));
        RO[nd][2] = __fadd_rn(RO[nd][2], half_lo(o0[1]));
        RO[nd][3] = __fadd_rn(RO[nd][3], half_hi(o0[1]));
        RO[nd + 1][0] = __fadd_rn(RO[nd + 1][0], half_lo(o1[0]));
        RO[nd + 1][1] = __fadd_rn(RO[nd + 1][1], half_hi(o1[0]));
        RO[nd + 1][2] = __fadd_rn(RO[nd + 1][2], half_lo(o1[1]));
        RO[nd + 1][3] = __fadd_rn(RO[nd + 1][3], half_hi(o1[1]));
      }
    }
    __syncthreads();  // the stage is refilled two iterations later
  }

  // epilogue: full denominators, FP32 reciprocal, V scale, BF16 store
  d0 = __fadd_rn(d0, __shfl_xor_sync(0xffffffffu, d0, 1));
  d0 = __fadd_rn(d0, __shfl_xor_sync(0xffffffffu, d0, 2));
  d1 = __fadd_rn(d1, __shfl_xor_sync(0xffffffffu, d1, 1));
  d1 = __fadd_rn(d1, __shfl_xor_sync(0xffffffffu, d1, 2));
  const float rc0 = __frcp_rn(d0), rc1 = __frcp_rn(d1);
  const float* vsc = p.v_scale + bh * D;
  const int ra = row0 + g, rb = row0 + g + 8;
#pragma unroll
  for (int nd = 0; nd < D / 8; ++nd) {
    const int col = nd * 8 + 2 * c;
    const float s0 = vsc[col], s1 = vsc[col + 1];
    if (ra < p.N) {
      const uint32_t w = f32_to_bf16_rn(__fmul_rn(__fmul_rn(RO[nd][0], rc0), s0)) |
                         ((uint32_t)f32_to_bf16_rn(__fmul_rn(__fmul_rn(RO[nd][1], rc0), s1)) << 16);
      *reinterpret_cast<uint32_t*>(p.out + b * p.os_b + (int64_t)ra * p.os_n + h * p.os_h + col) = w;
    }
    if (rb < p.N) {
      const uint32_t w = f32_to_bf16_rn(__fmul_rn(__fmul_rn(RO[nd][2], rc1), s0)) |
                         ((uint32_t)f32_to_bf16_rn(__fmul_rn(__fmul_rn(RO[nd][3], rc1), s1)) << 16);
      *reinterpret_cast<uint32_t*>(p.out + b * p.os_b + (int64_t)rb * p.os_n + h * p.os_h + col) = w;
    }
  }
}

// One tile of int32 scores through the same QK code (debug export).
template <int D>
__global__ void __launch_bounds__(kThreads, 1) debug_qk_mma_kernel(const AttnParams p, int b, int h,
                                                                   int qt, int kt, int32_t* s_out) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const size_t bh = (size_t)b * p.H + h;
  load_k<D>(sm, 0, p.k8 + bh * p.Nk * D, kt);  // scores only: no V tile (no V pointer)
  cp_async_commit();
  cp_async_wait<0>();
  __syncthreads();
  const int row0 = qt * kQTile + warp * 16;
  uint32_t qa[D / 32][4];
  const int8_t* q0 = p.q8 + (bh * p.Nq + row0 + g) * D;
  const int8_t* q1 = q0 + 8 * D;
#pragma unroll
  for (int ks = 0; ks < D / 32; ++ks) {
    qa[ks][0] = *reinterpret_cast<const uint32_t*>(q0 + ks * 32 + 4 * c);
    qa[ks][1] = *reinterpret_cast<const uint32_t*>(q1 + ks * 32 + 4 * c);
    qa[ks][2] = *reinterpret_cast<const uint32_t*>(q0 + ks * 32 + 16 + 4 * c);
    qa[ks][3] = *reinterpret_cast<const uint32_t*>(q1 + ks * 32 + 16 + 4 * c);
  }
  int32_t S[8][4];
  qk_tile<D>(sm, 0, qa, S);
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int row = warp * 16 + g + (r >> 1) * 8;
      s_out[row * kKTile + key_of(j, 2 * c + (r & 1))] = S[j][r];
    }
}

template <int D>
int launch(const AttnParams& p, cudaStream_t s) {
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto* fn = attn_mma_kernel<D>;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  fn<<<dim3(p.Nq / kQTile, p.H, p.B), kThreads, smem, s>>>(p);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

template <int D>
int launch_dbg(const AttnParams& p, int b, int h, int qt, int kt, int32_t* s_out, cudaStream_t s) {
  const size_t smem = sizeof(Smem<D>) + 1024;
  auto* fn = debug_qk_mma_kernel<D>;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  fn<<<1, kThreads, smem, s>>>(p, b, h, qt, kt, s_out);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

int launch_attn_mma(const AttnParams& p, cudaStream_t s) {
  if (p.D == 128) return launch<128>(p, s);
  if (p.D == 64) return launch<64>(p, s);
  return SAGE_ERR_UNSUPPORTED;
}

int launch_debug_qk_mma(const AttnParams& p, int b, int h, int q_tile, int k_tile, int32_t* s_out,
                        cudaStream_t s) {
  if (p.D == 128) return launch_dbg<128>(p, b, h, q_tile, k_tile, s_out, s);
  if (p.D == 64) return launch_dbg<64>(p, b, h, q_tile, k_tile, s_out, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
