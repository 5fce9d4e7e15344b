// tcgen05 / TMA / mbarrier primitives, the softmax helpers of one 64-key
// tile, and tensor-map encoding, shared by the sm_100a mainloops.
#pragma once
#include <cuda.h>

#include "sage_common.cuh"

namespace sage {
namespace tc {

// ------------------------------------------------------------- primitives
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b)) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(b)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{.reg .pred p; mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2; selp.u32 %0, 1, 0, p;}"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}

// The slow path of a bounded wait, kept out of line: inlined at every wait
// it made the mainloops' hot code several times larger.
static __device__ __noinline__ bool wait_slow(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                              DeviceStatus* st, int where, long long limit, bool honour_abort) {
  const long long t0 = clock64();
  for (uint32_t i = 0;; ++i) {
    if (mbar_try(b, parity)) return true;
    if ((i & 31u) == 31u) {
      if (honour_abort && *abort_flag) return false;
      if (clock64() - t0 > limit) break;
    }
  }
  *abort_flag = 1;
  if (st && atomicCAS(&st->code, 0, (int)SAGE_ERR_TIMEOUT) == 0) {
    st->where = where;
    st->block = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
  }
  return false;
}
// Bounded wait.  Returns false if the CTA is aborting or the wait ran out
// (then the status word and the abort flag are set).  A phase that is
// already complete costs one try_wait.
__device__ __forceinline__ bool wait_bounded(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                             DeviceStatus* st, int where, long long limit,
                                             bool honour_abort = true) {
  if (mbar_try(b, parity)) return true;
  return wait_slow(b, parity, abort_flag, st, where, limit, honour_abort);
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_commit(uint64_t* b) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(b))
               : "memory");
}

// Shared-memory matrix descriptor of a K-major tile whose rows are
// `row_bytes` (64 or 128) long, written by TMA with the matching swizzle:
// 8-row core groups `8 * row_bytes` apart (stride byte offset), leading
// byte offset unused for swizzled K-major layouts, descriptor version 1.
__device__ __forceinline__ uint64_t smem_desc(const void* tile, int row_bytes) {
  const uint32_t a = smem_u32(tile);
  uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
  d |= (uint64_t)1u << 16;                                   // LBO (16 B), ignored
  d |= (uint64_t)(((8u * row_bytes) >> 4) & 0x3FFFu) << 32;  // SBO
  d |= (uint64_t)1u << 46;                                   // version
  d |= (uint64_t)(row_bytes == 128 ? 2u : 4u) << 61;         // SWIZZLE_128B / SWIZZLE_64B
  return d;
}

// Instruction descriptors: M = 128, K-major A and B.
// QK: INT8 x INT8 -> S32, N keys.  PV: E4M3 x E4M3 -> F16, N = D.
__host__ __device__ constexpr uint32_t idesc_qk(int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(kQTile >> 4) << 24);
}
template <int D>
__host__ __device__ constexpr uint32_t idesc_pv() {
  return ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kQTile >> 4) << 24);
}
// PV with an FP32 accumulator (c_format = F32).
template <int D>
__host__ __device__ constexpr uint32_t idesc_pv_f32() {
  return (1u << 4) | ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kQTile >> 4) << 24);
}

__device__ __forceinline__ void mma_i8_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{.reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void mma_f8_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{.reg .pred p; setp.ne.b32 p, %4, 0; tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;}" ::"r"(
          d_tmem),
      "r"(a_tmem), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 lanes x 64 columns of 32 bits -> 64 registers (thread t = lane base + t).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,"
      "%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, "
      "[%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]),
        "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]),
        "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]),
        "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]),
        "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
// 32 columns of FP16 values -> 16 registers, two per register.
__device__ __forceinline__ void tmem_ld16_pack16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.pack::16b.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 columns of 32 bits -> 16 registers.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// Wait for this thread's TMEM loads; the registers pass through the wait so
// that no use of them can be scheduled before it.
__device__ __forceinline__ void tmem_wait_ld16(uint32_t (&r)[16]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_free(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols) : "memory");
}


// ------------------------------------------------------------- softmax helpers
// Tile maximum fl32(max(S) * c) of one row's 64 scores (the max of the
// integers is exact, and rounding is monotone with c >= 0); TAIL masks keys
// >= nvalid.
template <bool TAIL>
__device__ __forceinline__ float tile_max(const uint32_t (&S)[64], float cs, int nvalid) {
  // a tree of three-input integer maxima: 64 -> 22 -> 8 -> 3 -> 1
  int v[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) v[j] = (TAIL && j >= nvalid) ? INT_MIN : (int)S[j];
  int a[22], b[8];
#pragma unroll
  for (int j = 0; j < 21; ++j) a[j] = __vimax3_s32(v[3 * j], v[3 * j + 1], v[3 * j + 2]);
  a[21] = v[63];
#pragma unroll
  for (int j = 0; j < 7; ++j) b[j] = __vimax3_s32(a[3 * j], a[3 * j + 1], a[3 * j + 2]);
  b[7] = a[21];
  const int m = __vimax3_s32(__vimax3_s32(b[0], b[1], b[2]), __vimax3_s32(b[3], b[4], b[5]), max(b[6], b[7]));
  return __fmul_rn(__int2float_rn(m), cs);
}

// Probabilities of 16 of a row's keys (k0..k0+15) against the running max:
// p = 2^(fl32(S*c - m_new)) in FP32 into the partial sums rs, E4M3 bytes (key
// order from the low byte) into P[k0/4 ..].  The exponent argument is one
// fused multiply-add on the exact float of S (|S| < 2^22, so the conversion
// is exact).  Scalar operations and this statement order measured fastest of
// the exact forms tried (packed FP32x2 pairs, a float image with a packed or
// scalar unbias).
template <bool TAIL>
__device__ __forceinline__ void chunk_exp(const uint32_t (&Sc)[16], int k0, float cs, float nm, int nvalid,
                                          float (&rs)[4], uint32_t (&P)[16]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; e += 2) {
      const int j = 4 * q + e;
      pv[e] = __fmaf_rn(__int2float_rn((int32_t)Sc[j]), cs, nm);
      pv[e + 1] = __fmaf_rn(__int2float_rn((int32_t)Sc[j + 1]), cs, nm);
      pv[e] = ex2(pv[e]);
      pv[e + 1] = ex2(pv[e + 1]);
      if (TAIL && k0 + j >= nvalid) pv[e] = 0.0f;
      if (TAIL && k0 + j + 1 >= nvalid) pv[e + 1] = 0.0f;
    }
    rs[0] = __fadd_rn(rs[0], pv[0]);
    rs[1] = __fadd_rn(rs[1], pv[1]);
    rs[2] = __fadd_rn(rs[2], pv[2]);
    rs[3] = __fadd_rn(rs[3], pv[3]);
    asm("{.reg .b16 lo, hi; cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1; cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;"
        " mov.b32 %0, {lo, hi};}"
        : "=r"(P[k0 / 4 + q])
        : "f"(pv[0]), "f"(pv[1]), "f"(pv[2]), "f"(pv[3]));
  }
}

// The exponential pass over a tile: the scores are read again from TMEM in
// four 16-column chunks (double-buffered), so that the registers of the max
// pass are free.  Returns the FP32 row sum.  The load of the first chunk into
// A has already been issued (tmem_ld16(taddr, A)) by the caller.
template <bool TAIL>
__device__ __forceinline__ float tile_exp_issued(uint32_t taddr, float cs, float m_new, int nvalid,
                                                 uint32_t (&P)[16], uint32_t (&A)[16]) {
  const float nm = -m_new;
  float rs[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  uint32_t Bc[16];
  tmem_wait_ld16(A);
  tmem_ld16(taddr + 16, Bc);
  chunk_exp<TAIL>(A, 0, cs, nm, nvalid, rs, P);
  tmem_wait_ld16(Bc);
  tmem_ld16(taddr + 32, A);
  chunk_exp<TAIL>(Bc, 16, cs, nm, nvalid, rs, P);
  tmem_wait_ld16(A);
  tmem_ld16(taddr + 48, Bc);
  chunk_exp<TAIL>(A, 32, cs, nm, nvalid, rs, P);
  tmem_wait_ld16(Bc);
  chunk_exp<TAIL>(Bc, 48, cs, nm, nvalid, rs, P);
  return __fadd_rn(__fadd_rn(rs[0], rs[1]), __fadd_rn(rs[2], rs[3]));
}

template <bool TAIL>
__device__ __forceinline__ float tile_exp(uint32_t taddr, float cs, float m_new, int nvalid, uint32_t (&P)[16]) {
  uint32_t A[16];
  tmem_ld16(taddr, A);
  return tile_exp_issued<TAIL>(taddr, cs, m_new, nvalid, P, A);
}

// ------------------------------------------------------------- tensor maps
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// Looked up once per process; the initialisation of a function-local static
// is thread-safe, so concurrent first calls all see the same result.
inline EncodeTiledFn encode_fn() {
  static const EncodeTiledFn fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(f);
    return EncodeTiledFn(nullptr);
  }();
  return fn;
}

// 3-D uint8 tensor map: dims {inner, rows, BH} with row pitch `pitch` bytes
// and head pitch `hpitch` bytes; box {box_inner, box_rows, 1}.
inline bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t bh, uint64_t pitch,
              uint64_t hpitch, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {inner, rows, bh};
  const cuuint64_t strides[2] = {pitch, hpitch};
  const cuuint32_t box[3] = {box_inner, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = box_inner == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace tc
}  // namespace sage
