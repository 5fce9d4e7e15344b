// Fused attention mainloop on 5th-generation tensor cores (tcgen05, TMEM,
// TMA), sm_100a.
//
// One CTA = one 128-row query tile of one (b, h); nineteen warps with fixed
// roles (the ownership split of the pages' VEA-B design, built on TMEM):
//   warps 0-7   QK/softmax owners.  Warp w owns query rows 32*(w%4)..+31
//               (TMEM lanes of its quadrant) for the 64-key tiles t with
//               t % 2 == w / 4, so two warps of a quadrant work on
//               consecutive tiles at once.  Per tile a warp reads the int32
//               scores from TMEM, takes the tile max, receives the running
//               max m(t-1) from its partner (shared memory + mbarrier), hands
//               m(t) on, computes the rescale factor r, the FP32
//               probabilities, its part of the denominator, and writes the
//               E4M3 probabilities back to TMEM over the scores.
//   warps 8-15  output owners: thread (w, lane) owns half of the FP32 output
//               row RO of row 32*(w%4)+lane in registers.  Per tile it waits
//               for the first FP16 K32 buffer, reads r, applies it, then adds
//               each buffer (read from TMEM) in order, releasing both with
//               one arrival once the second is in registers; at the end it
//               applies 1/d and the V scale and stores BF16.
//   warp 16     TMA producer: the Q tile once, then K and V^T stages of 128
//               keys (two tiles) into a ring of shared-memory stages.
//   warp 17     QK issuer: per 128-key group four INT8 MMAs (N = 128, K = 32
//               each) into one of two TMEM score buffers.
//   warp 18     PV issuer: once a tile's probabilities are in and both FP16
//               buffers of the previous tile have been read (one barrier),
//               per K32 slice one E4M3 MMA, with the probabilities as the TMEM
//               A operand, into an FP16 accumulator that starts at zero (the
//               instantaneous buffer), one TMEM buffer per slice.
// The producer and issuer warps run their loops and waits with all 32 lanes
// (lane 0 issues the copies, MMAs, commits and arrivals), which keeps them off
// the slow divergent path.  Each wait there is followed by __syncwarp, so lane
// 0 acts only after every lane has seen the phase; as every next phase of
// those barriers needs an action of lane 0, the phase stays complete while
// any lane still polls, and all lanes reach the same outcome.
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
// The denominator is kept as two partial sums, one per softmax warp of a
// quadrant, each rescaled to the running max of its latest tile and merged
// at the end; the pages leave its summation order open.
#include <cuda.h>

#include <type_traits>

#include "sage_common.cuh"
#include "tc_prims.cuh"

namespace sage {
namespace {

using namespace tc;

constexpr int kThreadsTC = 608;
constexpr int kSoftWarp0 = 0;  // warps 0-7: softmax owners
constexpr int kOutWarp0 = 8;   // warps 8-15: output owners
constexpr int kLoadWarp = 16;
constexpr int kQkWarp = 17;    // QK issuer; also allocates and frees the tensor memory
constexpr int kPvWarp = 18;    // PV issuer
constexpr int kGroup = 128;    // keys per K/V stage and per QK MMA (two 64-key tiles)
constexpr int kStages = 3;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;      // two int32 score buffers of 128 columns (one group each); the
                                   // E4M3 P of a tile overlays the first 16 columns of its 64
constexpr uint32_t kColO = 256;    // two FP16 PV buffers of 128 columns (one per K32 slice)

template <int D>
struct TcSmem {
  alignas(1024) uint8_t q[kQTile * D];
  alignas(1024) uint8_t k[kStages][kGroup * D];
  alignas(1024) uint8_t v[kStages][D * kGroup];
  float r_ring[2][kQTile];
  float m_x[2][kQTile];               // running max after a tile, for the partner warp
  float m_fin[2][kQTile], d_fin[2][kQTile];
  float rcp[kQTile];
  uint64_t q_full;
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], r_free[2];
  uint64_t o_full[2], o_free;  // o_free: both FP16 buffers of a tile have been read
  uint64_t m_full[4][2];
  uint64_t fin, done;
  uint64_t drain_qk, drain_pv;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__device__ __forceinline__ TcSmem<D>& tc_smem() {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  return *reinterpret_cast<TcSmem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
}

// ------------------------------------------------------------------ kernel
// DBG (the score export sage_debug_qk_s32): a one-CTA launch for query tile
// p.dbg_qt of head (p.dbg_b, p.dbg_h) that runs the whole mainloop and also
// copies the int32 scores of key tile p.dbg_tile, as its softmax owners read
// them from TMEM, to p.dbg_out (128 x 64, row-major); it stores no output.
template <int D, bool DBG>
__global__ void __launch_bounds__(kThreadsTC, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  constexpr int DH = D / 2;  // output columns owned by one output thread
  TcSmem<D>& sm = tc_smem<D>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = DBG ? p.dbg_qt : (int)blockIdx.x;
  const int h = DBG ? p.dbg_h : (int)blockIdx.y;
  const int b = DBG ? p.dbg_b : (int)blockIdx.z;
  const int bh = b * p.H + h;
  const int T = p.T64;            // 64-key tiles
  const int G = (T + 1) >> 1;     // 128-key groups
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 1);
      mbar_init(&sm.p_full[i], kQTile);
      mbar_init(&sm.r_free[i], 2 * kQTile + 1);  // output owners and the PV issuer
      mbar_init(&sm.o_full[i], 1);
      for (int q = 0; q < 4; ++q) mbar_init(&sm.m_full[q][i], 32);
    }
    mbar_init(&sm.o_free, 2 * kQTile);
    mbar_init(&sm.fin, 2 * kQTile);
    mbar_init(&sm.done, kQTile);
    mbar_init(&sm.drain_qk, 1);
    mbar_init(&sm.drain_pv, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kQkWarp) tmem_alloc(&sm.tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // Launched as a programmatic dependent of the prepass: the set-up above
  // overlaps its last CTAs; nothing the prepass writes is read before this
  // returns (the prepass grid complete, its writes visible).
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp >= kSoftWarp0 && warp < kOutWarp0) {
    // ------------------------------------------------ QK / softmax owners
    const int quad = warp & 3, par = (warp - kSoftWarp0) >> 2;  // rows 32*quad.., tiles t % 2 == par
    const int i = quad * 32 + lane;              // row within the tile = TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int row = qt * kQTile + i;
    const int grp = row / kQGroup;
    const float qs = grp < p.G32 ? p.q_scale[(size_t)bh * p.G32 + grp] : 0.0f;
    const float* ksc = p.k_scale + (size_t)bh * T;
    const int ntail = p.N - (T - 1) * kKTile;  // valid keys of the last tile
    float m_own = -INFINITY, d_own = 0.0f;     // this warp's latest running max and partial denominator
    float ks_next = par < T ? ksc[par] : 0.0f;  // K scale of this warp's next tile, loaded a tile ahead
    // one 64-key tile t of this warp (TAIL: the ragged last tile, keys >= ntail
    // masked); returns false if a wait gave up
    auto tile_step = [&](auto tail_tag, int t) -> bool {
      constexpr bool TAIL = decltype(tail_tag)::value;
      const int g = t >> 1, sb = g & 1;
      const uint32_t cols = kColS + 128 * sb + 64 * par;
      const float ks = ks_next;
      if (t + 2 < T) ks_next = ksc[t + 2];
      if (!wait_bounded(&sm.s_full[sb], (uint32_t)((g >> 1) & 1), abort_flag, p.status, 1, p.wait_limit)) return false;
      tc_fence_after();
      uint32_t S[64];
      tmem_ld64(lane_addr + cols, S);
      tmem_wait_ld();
      if (DBG && t == p.dbg_tile) {
#pragma unroll
        for (int j = 0; j < 64; ++j) p.dbg_out[i * kKTile + j] = (int32_t)S[j];
      }
      // test the handoffs of this tile early; their latency overlaps the max pass
      const bool m_ready = t == 0 || mbar_try(&sm.m_full[quad][par ^ 1], (uint32_t)(((t - 1) >> 1) & 1));
      const bool r_ready = mbar_try(&sm.r_free[par], (uint32_t)(((t >> 1) & 1) ^ 1));
      const float cs = __fmul_rn(__fmul_rn(qs, ks), p.sl2);
      const float tmax = tile_max<TAIL>(S, cs, ntail);
      // at D = 64 the first chunk of the exponential pass is requested here,
      // so that its TMEM latency overlaps the handoff of the running max (at
      // D = 128 the extra live registers spill and the step is 9% slower)
      [[maybe_unused]] uint32_t A0[16];
      if constexpr (D == 64) tmem_ld16(lane_addr + cols, A0);
      // running max: m(t) = max(m(t-1), tile max), m(t-1) from the partner warp
      float m_prev = -INFINITY;
      if (t > 0) {
        if (!m_ready && !wait_bounded(&sm.m_full[quad][par ^ 1], (uint32_t)(((t - 1) >> 1) & 1), abort_flag,
                                      p.status, 15, p.wait_limit))
          return false;
        m_prev = sm.m_x[par ^ 1][i];
      }
      const float m_new = fmaxf(m_prev, tmax);
      sm.m_x[par][i] = m_new;
      mbar_arrive(&sm.m_full[quad][par]);
      const float r = (m_new == m_prev) ? 1.0f : ex2(__fsub_rn(m_prev, m_new));
      uint32_t P[16];
      float rs;
      if constexpr (D == 64)
        rs = tile_exp_issued<TAIL>(lane_addr + cols, cs, m_new, ntail, P, A0);
      else
        rs = tile_exp<TAIL>(lane_addr + cols, cs, m_new, ntail, P);
      // this warp's partial denominator, carried from its previous tile's max
      d_own = (m_own == m_new) ? __fadd_rn(d_own, rs) : __fadd_rn(__fmul_rn(d_own, ex2(__fsub_rn(m_own, m_new))), rs);
      m_own = m_new;
      tmem_st16(lane_addr + cols, P);  // E4M3 P over the first 16 score columns of the tile
      tmem_wait_st();
      if (!r_ready &&
          !wait_bounded(&sm.r_free[par], (uint32_t)(((t >> 1) & 1) ^ 1), abort_flag, p.status, 2, p.wait_limit))
        return false;
      sm.r_ring[par][i] = r;
      tc_fence_before();
      mbar_arrive(&sm.p_full[par]);
      return true;
    };
    // the loop holds one copy of the tile code; a ragged last tile is peeled
    // off after it, so the masked copy stays out of the hot loop
    const int t_full = ntail == kKTile ? T : T - 1;  // tiles without masking
    bool ok = true;
    int t = par;
    for (; ok && t < t_full; t += 2) ok = tile_step(std::false_type{}, t);
    if (ok && t == T - 1 && t_full < T) tile_step(std::true_type{}, t);
    // merge the two partial denominators at the final running max
    sm.m_fin[par][i] = m_own;
    sm.d_fin[par][i] = d_own;
    mbar_arrive(&sm.fin);
    if (par == 0) {
      if (wait_bounded(&sm.fin, 0, abort_flag, p.status, 16, p.wait_limit)) {
        const float m0 = sm.m_fin[0][i], m1 = sm.m_fin[1][i];
        const float mf = fmaxf(m0, m1);
        const float d0 = m0 == mf ? sm.d_fin[0][i] : __fmul_rn(sm.d_fin[0][i], ex2(__fsub_rn(m0, mf)));
        const float d1 = m1 == mf ? sm.d_fin[1][i] : __fmul_rn(sm.d_fin[1][i], ex2(__fsub_rn(m1, mf)));
        sm.rcp[i] = __frcp_rn(__fadd_rn(d0, d1));
      }
      mbar_arrive(&sm.done);
    }
  } else if (warp < kLoadWarp) {
    // ---------------------------------------- output owners (half rows)
    const int quad = warp & 3;
    const int i = quad * 32 + lane;                  // row within the tile
    const int c_base = warp < kOutWarp0 + 4 ? 0 : DH;  // this thread's output columns
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    float RO[DH];
#pragma unroll
    for (int c = 0; c < DH; ++c) RO[c] = 0.0f;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int bi = t & 1;
      // slice 0 first: its MMA was issued after this tile's probabilities were
      // in, so p_full(t) is complete by then and its wait below is one test
      // (one wake-up of this warp per tile)
      if (!wait_bounded(&sm.o_full[0], (uint32_t)(t & 1), abort_flag, p.status, 4, p.wait_limit)) break;
      if (!wait_bounded(&sm.p_full[bi], (uint32_t)((t >> 1) & 1), abort_flag, p.status, 3, p.wait_limit)) break;
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
      for (int sl = 0; sl < 2; ++sl) {  // K32 slice sl of tile t sits in buffer sl
        if (sl == 1 && !wait_bounded(&sm.o_full[1], (uint32_t)(t & 1), abort_flag, p.status, 4, p.wait_limit)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 32 columns at a time (16 registers of FP16 pairs); both buffers are
        // released once the last columns of slice 1 are in registers (slice
        // 0 was read before, so one arrival per tile covers both)
#pragma unroll
        for (int c0 = 0; c0 < DH; c0 += 32) {
          uint32_t hv[16];
          tmem_ld16_pack16(lane_addr + kColO + 128 * sl + c_base + c0, hv);
          tmem_wait_ld();
          if (sl == 1 && c0 + 32 >= DH) {
            tc_fence_before();
            mbar_arrive(&sm.o_free);  // both buffers may be overwritten now
          }
          // RO += float(tmp), one rounding per element (float(tmp) is exact):
          // one mixed-precision add (FP16 operand, FP32 accumulator) each
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            asm("{.reg .b16 lo, hi; mov.b32 {lo, hi}, %2; add.rn.f32.f16 %0, lo, %0; add.rn.f32.f16 %1, hi, %1;}"
                : "+f"(RO[c0 + 2 * j]), "+f"(RO[c0 + 2 * j + 1])
                : "r"(hv[j]));
          }
        }
      }
    }
    if (!DBG && ok && wait_bounded(&sm.done, 0, abort_flag, p.status, 5, p.wait_limit) && !*abort_flag) {
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
    // The whole warp runs the loop and the waits; lane 0 issues the copies.
    const bool leader = lane == 0;
    int issued = 0;
    if (leader) {
      mbar_expect_tx(&sm.q_full, kQTile * D);
      tma_load_3d(sm.q, &tm_q, 0, qt * kQTile, bh, &sm.q_full);
    }
    for (int g = 0; g < G; ++g) {
      const int st = g % kStages;
      const bool ok =
          wait_bounded(&sm.kv_empty[st], (uint32_t)(((g / kStages) & 1) ^ 1), abort_flag, p.status, 6, p.wait_limit);
      __syncwarp();  // every lane has seen the phase before lane 0 acts on it
      if (!ok) break;
      if (p.stall_tile >= 0 && p.stall_tile / 2 == g) continue;  // test hook: this stage never arrives
      if (leader) {
        mbar_expect_tx(&sm.kv_full[st], 2 * kGroup * D);
        tma_load_3d(sm.k[st], &tm_k, 0, g * kGroup, bh, &sm.kv_full[st]);
        tma_load_3d(sm.v[st], &tm_v, g * kGroup, 0, bh, &sm.kv_full[st]);
      }
      issued = g + 1;
    }
    // leave no copy in flight: wait for every issued stage and for Q
    wait_bounded(&sm.q_full, 0, abort_flag, nullptr, 7, p.wait_limit, false);
    for (int u = max(0, issued - kStages); u < issued; ++u)
      if (!(p.stall_tile >= 0 && p.stall_tile / 2 == u))
        wait_bounded(&sm.kv_full[u % kStages], (uint32_t)((u / kStages) & 1), abort_flag, nullptr, 8,
                     p.wait_limit, false);
  } else if (warp == kQkWarp) {
    // ----------------------------------------------------------- QK issuer
    // The whole warp runs the loop and the waits; lane 0 issues and commits.
    const bool leader = lane == 0;
    const uint32_t iqk = idesc_qk(kGroup);
    const uint64_t qdesc = smem_desc(sm.q, D);
    bool ok = wait_bounded(&sm.q_full, 0, abort_flag, p.status, 9, p.wait_limit);
    __syncwarp();
    for (int g = 0; ok && g < G; ++g) {
      const int st = g % kStages, sb = g & 1;
      // the buffer's last probabilities (group g - 2) have been read by PV
      ok = wait_bounded(&sm.s_free[sb], (uint32_t)(((g >> 1) & 1) ^ 1), abort_flag, p.status, 11, p.wait_limit) &&
           wait_bounded(&sm.kv_full[st], (uint32_t)((g / kStages) & 1), abort_flag, p.status, 10, p.wait_limit);
      __syncwarp();  // every lane has seen the phases before lane 0 acts on them
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint64_t kdesc = smem_desc(sm.k[st], D);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + kColS + 128 * sb, qdesc + 2 * kk, kdesc + 2 * kk, iqk, kk > 0);
        tc_commit(&sm.s_full[sb]);
      }
    }
    // no MMA may still be writing TMEM when it is freed
    __syncwarp();
    if (leader) tc_commit(&sm.drain_qk);
    __syncwarp();
    wait_bounded(&sm.drain_qk, 0, abort_flag, nullptr, 14, p.wait_limit, false);
  } else if (warp == kPvWarp) {
    // ----------------------------------------------------------- PV issuer
    // The whole warp runs the loop and the waits; lane 0 issues, commits and arrives.
    const bool leader = lane == 0;
    const uint32_t ipv = idesc_pv<D>();
    for (int t = 0; t < T; ++t) {
      const int g = t >> 1, sb = g & 1, st = g % kStages, half = t & 1;
      // this tile's probabilities; the V^T stage, which arrived with the K stage
      // the QK issuer waited for; both FP16 buffers read by the output owners
      // (one wait: a single wake-up of this warp per tile)
      const bool ok =
          wait_bounded(&sm.p_full[half], (uint32_t)((t >> 1) & 1), abort_flag, p.status, 12, p.wait_limit) &&
          (half == 1 ||
           wait_bounded(&sm.kv_full[st], (uint32_t)((g / kStages) & 1), abort_flag, p.status, 18, p.wait_limit)) &&
          wait_bounded(&sm.o_free, (uint32_t)((t & 1) ^ 1), abort_flag, p.status, 13, p.wait_limit);
      __syncwarp();  // every lane has seen the phases before lane 0 acts on them
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        // seen: the softmax owners may complete this p_full slot again (tile t + 2)
        mbar_arrive(&sm.r_free[half]);
        // this tile's 64 keys within the stage's 128-byte V^T rows
        const uint64_t vdesc = smem_desc(sm.v[st], kGroup) + 4 * half;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl) {
          mma_f8_ts(tmem + kColO + 128 * sl, tmem + kColS + 128 * sb + 64 * half + 8 * sl, vdesc + 2 * sl, ipv, 0);
          tc_commit(&sm.o_full[sl]);
        }
        if (half == 1 || t + 1 == T) {  // the group's probabilities and K/V stage are consumed
          tc_commit(&sm.s_free[sb]);
          tc_commit(&sm.kv_empty[st]);
        }
      }
    }
    __syncwarp();
    if (leader) tc_commit(&sm.drain_pv);
    __syncwarp();
    wait_bounded(&sm.drain_pv, 0, abort_flag, nullptr, 17, p.wait_limit, false);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kQkWarp) tmem_free(tmem, kTmemCols);
}

// ------------------------------------------------------------------- host
template <int D>
size_t smem_bytes() {
  // at least 120 KB so that a second CTA (and its 512-column TMEM request)
  // never shares the SM
  const size_t need = sizeof(TcSmem<D>) + 1024;
  return need > 120 * 1024 ? need : 120 * 1024;
}

template <int D, bool DBG>
int launch_tc(const AttnParams& p, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const uint64_t bh = (uint64_t)p.B * p.H;
  if (!make_map(&mq, p.q8, D, p.Nq, bh, D, (uint64_t)p.Nq * D, D, kQTile) ||
      !make_map(&mk, p.k8, D, p.Nk, bh, D, (uint64_t)p.Nk * D, D, kGroup) ||
      !make_map(&mv, p.v8, p.Nk, D, bh, p.Nk, (uint64_t)D * p.Nk, kGroup, D))
    return SAGE_ERR_CUDA;
  auto* fn = attn_tc_kernel<D, DBG>;
  const size_t smem = smem_bytes<D>();
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = DBG ? dim3(1, 1, 1) : dim3(p.Nq / kQTile, p.H, p.B);
  cfg.blockDim = dim3(kThreadsTC);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  // programmatic dependent launch: the CTAs may start while the previous
  // kernel of the stream drains, once every CTA of that kernel has signalled
  // (the prepass kernels do at their start; others at their end)
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fn, mq, mk, mv, p) == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

bool tc_available() {
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return false;
  return major == 10 && encode_fn() != nullptr;
}

int launch_attn_tc(const AttnParams& p, cudaStream_t s) {
  if (p.D == 128) return p.dbg_out ? launch_tc<128, true>(p, s) : launch_tc<128, false>(p, s);
  if (p.D == 64) return p.dbg_out ? launch_tc<64, true>(p, s) : launch_tc<64, false>(p, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
