// Fused attention mainloop on 5th-generation tensor cores (tcgen05, TMEM,
// TMA), sm_100a.
//
// One CTA = one 128-row query tile of one (b, h); fifteen warps with fixed
// roles (the ownership split of the pages' VEA-B design, built on TMEM):
//   warps 0-3   QK/softmax owners: thread i owns query row i (TMEM lane i),
//               its running max m and denominator d.  Per tile they read the
//               int32 scores from TMEM, scale them, update m, d and the
//               rescale factor r, and write the E4M3 probabilities back to
//               TMEM over the scores they replace.
//   warps 4-11  output owners: thread (w, lane) owns half of the FP32 output
//               row RO of row 32*(w%4)+lane in registers.  Per tile it applies
//               r, then adds each FP16 K32 buffer (read from TMEM) in order;
//               at the end it applies 1/d and the V scale and stores BF16.
//   warp 12     TMA producer: the Q tile once, then K and V^T tiles of 64 keys
//               into a ring of shared-memory stages.
//   warp 13     QK issuer (one thread): per tile four INT8 MMAs (K = 32 each)
//               into one of two TMEM score buffers, up to two tiles ahead.
//   warp 14     PV issuer (one thread): per K32 slice one E4M3 MMA, with the
//               probabilities as the TMEM A operand, into an FP16 accumulator
//               that starts at zero (the instantaneous buffer), taken from a
//               ring of three TMEM buffers.
// Handoffs are block-scope mbarriers; tcgen05.commit signals MMA completion.
// Every wait is bounded: a wait that runs out records SAGE_ERR_TIMEOUT in
// the status word, raises a CTA-wide abort flag, and every role then leaves
// its loop, drains what it has in flight, and the TMEM is freed.
//
// Operation: "State-Ownership Architecture Decision", section "Non-Negotiable
// Dataflow" (tiles in increasing order; per tile QK, score scaling, max
// update, denominator update, FP8 probability conversion, two K32 FP16 PV
// MMAs, FP32 RO addition) and the exact handoff record (E4M3 bytes and the
// FP32 ro_rescale cross from the QK owner to the PV owner; final FP32
// reciprocal, then V scale, then BF16); the VEA-B role table of the same
// page; step order from "Sage2 SM89 Temporal Pair Experiment", "Candidate".
#include <cuda.h>

#include "sage_common.cuh"

namespace sage {
namespace {

constexpr int kThreadsTC = 480;
constexpr int kLoadWarp = 12;
constexpr int kMmaWarp = 13;   // QK issuer; also allocates and frees the tensor memory
constexpr int kPvWarp = 14;    // PV issuer
constexpr int kOBufs = 3;      // ring of FP16 PV buffers (one K32 slice each)
constexpr int kStages = 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // two int32 score buffers of 64 columns (E4M3 P overlays them)
constexpr uint32_t kColO = 128;    // ring of kOBufs FP16 PV buffers of 128 columns

template <int D>
struct TcSmem {
  alignas(1024) uint8_t q[kQTile * D];
  alignas(1024) uint8_t k[kStages][kKTile * D];
  alignas(1024) uint8_t v[kStages][D * kKTile];
  float r_ring[2][kQTile];
  float rcp[kQTile];
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], r_free[2];
  uint64_t o_full[kOBufs], o_free[kOBufs];
  uint64_t ro_ready, id_done;
  uint64_t done, drain, drain2;
  uint32_t tmem_base;
  int abort_flag;
};

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

// Bounded wait.  Returns false if the CTA is aborting or the wait ran out
// (then the status word and the abort flag are set).
__device__ __forceinline__ bool wait_bounded(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                             DeviceStatus* st, int where, long long limit,
                                             bool honour_abort = true) {
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
// QK: INT8 x INT8 -> S32, N = 64.  PV: E4M3 x E4M3 -> F16, N = D.
__host__ __device__ constexpr uint32_t idesc_qk() {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kKTile >> 3) << 17) | ((uint32_t)(kQTile >> 4) << 24);
}
template <int D>
__host__ __device__ constexpr uint32_t idesc_pv() {
  return ((uint32_t)(D >> 3) << 17) | ((uint32_t)(kQTile >> 4) << 24);
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
#define SAGE_R32(r) "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), \
    "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),   \
    "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),              \
    "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),              \
    "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
#define SAGE_W32(r) "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), \
    "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]),            \
    "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]),          \
    "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
#define SAGE_REGS32 "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}"
#define SAGE_REGS32_1 "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32}"

// 64 columns of FP16 values (one per 32-bit column) -> 32 registers, two per
// register (column 2j in the low half).
__device__ __forceinline__ void tmem_ld32_pack16(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.pack::16b.b32 " SAGE_REGS32 ", [%32];"
               : SAGE_R32(r)
               : "r"(taddr));
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
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ void tmem_free(uint32_t base, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(base), "r"(cols) : "memory");
}

template <int D>
__device__ __forceinline__ TcSmem<D>& tc_smem() {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  return *reinterpret_cast<TcSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------------ kernel
// Softmax of one tile for one row (TAIL: keys >= nvalid are masked).
// In: S[64] int32 scores.  Out: P[16] packed E4M3 probabilities; updates
// m and d, returns r (the factor applied to the older RO and d).
template <bool TAIL>
__device__ __forceinline__ float softmax_tile(const uint32_t (&S)[64], float cs, int nvalid, float& m,
                                              float& d, uint32_t (&P)[16]) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23: float bits of (magic + S) are magic_bits + S
  float fb[64];
#pragma unroll
  for (int j = 0; j < 64; ++j) {
    fb[j] = __int_as_float((int32_t)S[j] + 0x4B400000);
    if (TAIL && j >= nvalid) fb[j] = -INFINITY;
  }
  // tile max over the exact float images of the scores (3-input max)
  float mx[22];
#pragma unroll
  for (int j = 0; j < 21; ++j) mx[j] = fmaxf(fmaxf(fb[3 * j], fb[3 * j + 1]), fb[3 * j + 2]);
  mx[21] = fb[63];
#pragma unroll
  for (int j = 0; j < 7; ++j) mx[j] = fmaxf(fmaxf(mx[3 * j], mx[3 * j + 1]), mx[3 * j + 2]);
  const float fmx = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                          fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[21])));
  // max of fl32(S*c) = fl32(max(S)*c) since rounding is monotone and c >= 0
  const float tmax = __fmul_rn(__fsub_rn(fmx, kMagic), cs);
  const float m_new = fmaxf(m, tmax);
  const float r = (m_new == m) ? 1.0f : ex2(__fsub_rn(m, m_new));
  m = m_new;
  // exponent argument s - m_new as one FMA on the float image:
  // fb*c - (magic*c + m_new), with magic*c + m_new rounded once
  const float kofs = __fmaf_rn(kMagic, cs, m_new);
  float rs[2] = {0.0f, 0.0f};
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    float pv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int j = 4 * q + e;
      pv[e] = ex2(__fmaf_rn(fb[j], cs, -kofs));
      if (TAIL && j >= nvalid) pv[e] = 0.0f;
    }
    // two independent packed FP32 sums (pairs of lanes of an f32x2 add)
    asm("{.reg .b64 a, b; mov.b64 a, {%0, %1}; mov.b64 b, {%2, %3}; add.rn.f32x2 a, a, b;"
        " mov.b64 {%0, %1}, a;}"
        : "+f"(rs[0]), "+f"(rs[1])
        : "f"(pv[0]), "f"(pv[1]));
    asm("{.reg .b64 a, b; mov.b64 a, {%0, %1}; mov.b64 b, {%2, %3}; add.rn.f32x2 a, a, b;"
        " mov.b64 {%0, %1}, a;}"
        : "+f"(rs[0]), "+f"(rs[1])
        : "f"(pv[2]), "f"(pv[3]));
    P[q] = (uint32_t)e4m3x2(pv[0], pv[1]) | ((uint32_t)e4m3x2(pv[2], pv[3]) << 16);
  }
  d = __fadd_rn(__fmul_rn(d, r), __fadd_rn(rs[0], rs[1]));
  return r;
}

template <int D>
__global__ void __launch_bounds__(kThreadsTC, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int DH = D / 2;  // output columns owned by one output thread
  TcSmem<D>& sm = tc_smem<D>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int bh = b * p.H + h;
  const int T = p.T64;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 2);  // released by both MMA issuers
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 1);
      mbar_init(&sm.p_full[i], kQTile);
      mbar_init(&sm.r_free[i], 2 * kQTile);
    }
    for (int i = 0; i < kOBufs; ++i) {
      mbar_init(&sm.o_full[i], 1);
      mbar_init(&sm.o_free[i], 2 * kQTile);
    }
    mbar_init(&sm.done, kQTile);
    mbar_init(&sm.drain, 1);
    mbar_init(&sm.drain2, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < 4) {
    // ------------------------------------------------ QK / softmax owners
    const int i = threadIdx.x;  // row within the tile = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const int row = qt * kQTile + i;
    const int grp = row / kQGroup;
    const float qs = grp < p.G32 ? p.q_scale[(size_t)bh * p.G32 + grp] : 0.0f;
    const float* ksc = p.k_scale + (size_t)bh * T;
    const int ntail = p.N - (T - 1) * kKTile;  // valid keys of the last tile
    float m = -INFINITY, d = 0.0f;
    float ks_next = ksc[0];
    for (int t = 0; t < T; ++t) {
      const int bi = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      const float ks = ks_next;
      if (t + 1 < T) ks_next = ksc[t + 1];
      if (!wait_bounded(&sm.s_full[bi], ph, abort_flag, p.status, 1, p.wait_limit)) break;
      tc_fence_after();
      uint32_t S[64];
      tmem_ld64(lane_addr + kColS + 64 * bi, S);
      tmem_wait_ld();
      const float cs = __fmul_rn(__fmul_rn(qs, ks), p.sl2);
      uint32_t P[16];
      float r;
      if (t + 1 < T || ntail == kKTile) r = softmax_tile<false>(S, cs, kKTile, m, d, P);
      else r = softmax_tile<true>(S, cs, ntail, m, d, P);
      tmem_st16(lane_addr + kColS + 64 * bi, P);  // E4M3 P over the first 16 score columns
      tmem_wait_st();
      if (!wait_bounded(&sm.r_free[bi], ph ^ 1u, abort_flag, p.status, 2, p.wait_limit)) break;
      sm.r_ring[bi][i] = r;
      tc_fence_before();
      mbar_arrive(&sm.p_full[bi]);
    }
    sm.rcp[i] = __frcp_rn(d);
    mbar_arrive(&sm.done);
  } else if (warp < 12) {
    // ---------------------------------------- output owners (half rows)
    const int i = (warp & 3) * 32 + lane;      // row within the tile
    const int c_base = warp < 8 ? 0 : DH;      // this thread's output columns
    const uint32_t lane_addr = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    float RO[DH];
#pragma unroll
    for (int c = 0; c < DH; ++c) RO[c] = 0.0f;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int bi = t & 1;
      const uint32_t ph = (t >> 1) & 1;
      if (!wait_bounded(&sm.p_full[bi], ph, abort_flag, p.status, 3, p.wait_limit)) break;
      const float r = sm.r_ring[bi][i];
      mbar_arrive(&sm.r_free[bi]);
      if (r != 1.0f) {
#pragma unroll
        for (int c = 0; c < DH; c += 2) {
          asm("{.reg .b64 a, s; mov.b64 a, {%0, %1}; mov.b64 s, {%2, %2}; mul.rn.f32x2 a, a, s;"
              " mov.b64 {%0, %1}, a;}"
              : "+f"(RO[c]), "+f"(RO[c + 1])
              : "f"(r));
        }
      }
#pragma unroll
      for (int sl = 0; sl < 2; ++sl) {
        const int k = 2 * t + sl, ob = k % kOBufs;  // position in the buffer ring
        if (!wait_bounded(&sm.o_full[ob], (uint32_t)((k / kOBufs) & 1), abort_flag, p.status, 4, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t hv[DH / 2];
        if (DH == 64) {
          tmem_ld32_pack16(lane_addr + kColO + 128 * ob + c_base, *reinterpret_cast<uint32_t(*)[32]>(hv));
        } else {
          tmem_ld16_pack16(lane_addr + kColO + 128 * ob + c_base, *reinterpret_cast<uint32_t(*)[16]>(hv));
        }
        tmem_wait_ld();
        tc_fence_before();
        mbar_arrive(&sm.o_free[ob]);  // the buffer may be overwritten now
        // RO += float(tmp), one rounding per element (float(tmp) is exact):
        // widen the FP16 pair, then one packed FP32x2 add
#pragma unroll
        for (int j = 0; j < DH / 2; ++j) {
          asm("{.reg .b16 lo, hi; .reg .f32 a, b; .reg .b64 x, y;"
              " mov.b32 {lo, hi}, %2; cvt.f32.f16 a, lo; cvt.f32.f16 b, hi;"
              " mov.b64 x, {a, b}; mov.b64 y, {%0, %1}; add.rn.f32x2 y, y, x; mov.b64 {%0, %1}, y;}"
              : "+f"(RO[2 * j]), "+f"(RO[2 * j + 1])
              : "r"(hv[j]));
        }
      }
    }
    if (ok && wait_bounded(&sm.done, 0, abort_flag, p.status, 5, p.wait_limit) && !*abort_flag) {
      const int row = qt * kQTile + i;
      const float rc = sm.rcp[i];
      if (row < p.N) {
        const float* vs = p.v_scale + (size_t)bh * D + c_base;
        uint16_t* dst = p.out + b * p.os_b + (int64_t)row * p.os_n + h * p.os_h + c_base;
#pragma unroll
        for (int c = 0; c < DH; c += 8) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const uint32_t lo = f32_to_bf16_rn(__fmul_rn(__fmul_rn(RO[c + 2 * e], rc), vs[c + 2 * e]));
            const uint32_t hi = f32_to_bf16_rn(__fmul_rn(__fmul_rn(RO[c + 2 * e + 1], rc), vs[c + 2 * e + 1]));
            w[e] = lo | (hi << 16);
          }
          *reinterpret_cast<uint4*>(dst + c) = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
    }
  } else if (warp == kLoadWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued = 0;
      mbar_expect_tx(&sm.q_full, kQTile * D);
      tma_load_3d(sm.q, &tm_q, 0, qt * kQTile, bh, &sm.q_full);
      for (int t = 0; t < T; ++t) {
        const int st = t % kStages;
        if (!wait_bounded(&sm.kv_empty[st], (uint32_t)(((t / kStages) & 1) ^ 1), abort_flag, p.status, 6,
                          p.wait_limit))
          break;
        if (t == p.stall_tile) continue;  // test hook: this tile never arrives
        mbar_expect_tx(&sm.kv_full[st], 2 * kKTile * D);
        tma_load_3d(sm.k[st], &tm_k, 0, t * kKTile, bh, &sm.kv_full[st]);
        tma_load_3d(sm.v[st], &tm_v, t * kKTile, 0, bh, &sm.kv_full[st]);
        issued = t + 1;
      }
      // leave no copy in flight: wait for every issued stage and for Q
      wait_bounded(&sm.q_full, 0, abort_flag, nullptr, 7, p.wait_limit, false);
      for (int u = max(0, issued - kStages); u < issued; ++u)
        if (u != p.stall_tile)
          wait_bounded(&sm.kv_full[u % kStages], (uint32_t)((u / kStages) & 1), abort_flag, nullptr, 8,
                       p.wait_limit, false);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- QK issuer
    if (lane == 0) {
      const uint32_t iqk = idesc_qk();
      const uint64_t qdesc = smem_desc(sm.q, D);
      bool ok = wait_bounded(&sm.q_full, 0, abort_flag, p.status, 9, p.wait_limit);
      for (int t = 0; ok && t < T; ++t) {
        const int st = t % kStages, bi = t & 1;
        if (!wait_bounded(&sm.kv_full[st], (uint32_t)((t / kStages) & 1), abort_flag, p.status, 10, p.wait_limit))
          break;
        // PV(t-2) read its probabilities from this score buffer
        if (!wait_bounded(&sm.s_free[bi], (uint32_t)(((t >> 1) & 1) ^ 1), abort_flag, p.status, 11, p.wait_limit))
          break;
        tc_fence_after();
        const uint64_t kdesc = smem_desc(sm.k[st], D);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + kColS + 64 * bi, qdesc + 2 * kk, kdesc + 2 * kk, iqk, kk > 0);
        tc_commit(&sm.s_full[bi]);
        tc_commit(&sm.kv_empty[st]);
      }
      // no MMA may still be writing TMEM when it is freed
      tc_commit(&sm.drain);
      wait_bounded(&sm.drain, 0, abort_flag, nullptr, 14, p.wait_limit, false);
    }
    __syncwarp();
  } else if (warp == kPvWarp) {
    // ------------------------------------------------------- PV issuer
    if (lane == 0) {
      const uint32_t ipv = idesc_pv<D>();
      bool ok = true;
      for (int u = 0; ok && u < T; ++u) {
        const int bu = u & 1, su = u % kStages;
        // PV(u): two K32 slices, each into its own FP16 buffer from zero
        if (!wait_bounded(&sm.p_full[bu], (uint32_t)((u >> 1) & 1), abort_flag, p.status, 12, p.wait_limit)) break;
        // V(u) arrived with K(u) (already waited on by the QK issuer)
        if (!wait_bounded(&sm.kv_full[su], (uint32_t)((u / kStages) & 1), abort_flag, p.status, 16, p.wait_limit))
          break;
        tc_fence_after();
        const uint64_t vdesc = smem_desc(sm.v[su], kKTile);
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          const int k = 2 * u + sl, ob = k % kOBufs;
          if (!wait_bounded(&sm.o_free[ob], (uint32_t)(((k / kOBufs) & 1) ^ 1), abort_flag, p.status, 13,
                            p.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          mma_f8_ts(tmem + kColO + 128 * ob, tmem + kColS + 64 * bu + 8 * sl, vdesc + 2 * sl, ipv, 0);
          tc_commit(&sm.o_full[ob]);
        }
        if (!ok) break;
        tc_commit(&sm.s_free[bu]);
        tc_commit(&sm.kv_empty[su]);
      }
      tc_commit(&sm.drain2);
      wait_bounded(&sm.drain2, 0, abort_flag, nullptr, 15, p.wait_limit, false);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_free(tmem, kTmemCols);
}

// ------------------------------------------------ debug: one score tile
template <int D>
__global__ void __launch_bounds__(kThreadsTC, 1)
    debug_qk_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const AttnParams p, int b, int h, int qt, int kt, int32_t* s_out) {
  TcSmem<D>& sm = tc_smem<D>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = b * p.H + h;
  volatile int* abort_flag = &sm.abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    mbar_init(&sm.kv_full[0], 1);
    mbar_init(&sm.s_full[0], 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  if (warp == kLoadWarp && lane == 0) {
    mbar_expect_tx(&sm.q_full, kQTile * D);
    tma_load_3d(sm.q, &tm_q, 0, qt * kQTile, bh, &sm.q_full);
    mbar_expect_tx(&sm.kv_full[0], kKTile * D);
    tma_load_3d(sm.k[0], &tm_k, 0, kt * kKTile, bh, &sm.kv_full[0]);
    wait_bounded(&sm.q_full, 0, abort_flag, nullptr, 7, p.wait_limit, false);
    wait_bounded(&sm.kv_full[0], 0, abort_flag, nullptr, 8, p.wait_limit, false);
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      bool ok = wait_bounded(&sm.q_full, 0, abort_flag, p.status, 9, p.wait_limit) &&
                wait_bounded(&sm.kv_full[0], 0, abort_flag, p.status, 10, p.wait_limit);
      if (ok) {
        tc_fence_after();
        const uint64_t qdesc = smem_desc(sm.q, D), kdesc = smem_desc(sm.k[0], D);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + kColS, qdesc + 2 * kk, kdesc + 2 * kk, idesc_qk(), kk > 0);
      }
      tc_commit(&sm.s_full[0]);
      wait_bounded(&sm.s_full[0], 0, abort_flag, nullptr, 14, p.wait_limit, false);
    }
    __syncwarp();
  } else if (warp < 4) {
    if (wait_bounded(&sm.s_full[0], 0, abort_flag, p.status, 1, p.wait_limit) && !*abort_flag) {
      tc_fence_after();
      uint32_t S[64];
      tmem_ld64(tmem + ((uint32_t)(warp * 32) << 16) + kColS, S);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 64; ++j) s_out[threadIdx.x * kKTile + j] = (int32_t)S[j];
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_free(tmem, kTmemCols);
}

// ------------------------------------------------------------------- host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// 3-D uint8 tensor map: dims {inner, rows, BH} with row pitch `pitch` bytes
// and head pitch `hpitch` bytes; box {box_inner, box_rows, 1}.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint64_t bh, uint64_t pitch,
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

template <int D>
size_t smem_bytes() {
  // at least 120 KB so that a second CTA (and its 512-column TMEM request)
  // never shares the SM
  const size_t need = sizeof(TcSmem<D>) + 1024;
  return need > 120 * 1024 ? need : 120 * 1024;
}

template <int D>
int launch_tc(const AttnParams& p, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const uint64_t bh = (uint64_t)p.B * p.H;
  if (!make_map(&mq, p.q8, D, p.Nq, bh, D, (uint64_t)p.Nq * D, D, kQTile) ||
      !make_map(&mk, p.k8, D, p.Nk, bh, D, (uint64_t)p.Nk * D, D, kKTile) ||
      !make_map(&mv, p.v8, p.Nk, D, bh, p.Nk, (uint64_t)D * p.Nk, kKTile, D))
    return SAGE_ERR_CUDA;
  auto* fn = attn_tc_kernel<D>;
  const size_t smem = smem_bytes<D>();
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  fn<<<dim3(p.Nq / kQTile, p.H, p.B), kThreadsTC, smem, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

template <int D>
int launch_dbg_tc(const AttnParams& p, int b, int h, int qt, int kt, int32_t* s_out, cudaStream_t s) {
  CUtensorMap mq, mk;
  const uint64_t bh = (uint64_t)p.B * p.H;
  if (!make_map(&mq, p.q8, D, p.Nq, bh, D, (uint64_t)p.Nq * D, D, kQTile) ||
      !make_map(&mk, p.k8, D, p.Nk, bh, D, (uint64_t)p.Nk * D, D, kKTile))
    return SAGE_ERR_CUDA;
  auto* fn = debug_qk_tc_kernel<D>;
  const size_t smem = smem_bytes<D>();
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  fn<<<1, kThreadsTC, smem, s>>>(mq, mk, p, b, h, qt, kt, s_out);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

bool tc_available() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10 && encode_fn() != nullptr;
}

int launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  if (p.D == 128) return launch_tc<128>(p, s);
  if (p.D == 64) return launch_tc<64>(p, s);
  return SAGE_ERR_UNSUPPORTED;
}

int launch_debug_qk_tc(const AttnParams& p, int b, int h, int q_tile, int k_tile, int32_t* s_out,
                       cudaStream_t s) {
  if (p.D == 128) return launch_dbg_tc<128>(p, b, h, q_tile, k_tile, s_out, s);
  if (p.D == 64) return launch_dbg_tc<64>(p, b, h, q_tile, k_tile, s_out, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
