// Quality-gated fast mainloop on 5th-generation tensor cores, sm_100a.
//
// Same quantised inputs (INT8 Q/K with per-32/64-row scales, E4M3 V^T with
// per-channel scales) and the same INT8 QK^T and E4M3 probabilities as the
// exact mainloop, with two numerical departures that the pages assign to a
// future fast backend with its own contract ("vortex_fast": reordered
// reductions and a quality gate instead of exact parity; page "Vortex
// Exact", section "Scope"):
//   - the PV products are accumulated by the tensor core in FP32 in TMEM
//     across all tiles, instead of one FP16 buffer per K32 slice that is
//     added into an FP32 register accumulator;
//   - the softmax uses a "used" maximum per row that is raised only when a
//     tile's maximum exceeds it by more than kRescaleLog2 (so p <= 2^8, inside
//     the E4M3 range); the accumulator and the denominator are rescaled only
//     then, by correction warps that multiply the TMEM accumulator in place.
// Its results are held to a quality gate (cosine similarity against FP64
// attention, and distance from the exact path), not to oracle parity.
//
// One CTA = one 128-row query tile of one (b, h); fifteen warps:
//   warps 0-7   softmax owners, two per 32-row quadrant on alternate 64-key
//               tiles (as in the exact mainloop), handing the used maximum
//               to each other; per tile they write E4M3 P over the scores,
//               the rescale factor r and a per-quadrant "rescale" flag.
//   warps 8-11  correction and epilogue owners, one per quadrant: per tile
//               they wait for its probabilities and for the previous tile's
//               PV MMAs (one barrier per tile mod 4); on a tile whose flag is
//               set they scale the FP32 accumulator rows by r in TMEM and then
//               release that tile's PV MMAs; at the end they apply 1/d and the
//               V scale and store BF16.
//   warp 12     TMA producer (K and V^T stages of 128 keys).
//   warp 13     QK issuer (N = 128 per 128-key group, two score buffers).
//   warp 14     PV issuer: two E4M3 MMAs per tile (K32 slices) accumulating
//               into the FP32 TMEM accumulator.
// The producer and issuer warps run their loops with all 32 lanes and lane 0
// issues; every wait is bounded as in the exact mainloop.
#include <cuda.h>

#include <type_traits>

#include "sage_common.cuh"
#include "tc_prims.cuh"

namespace sage {
namespace {

using namespace tc;

constexpr int kThreadsF = 480;
constexpr int kCorrWarp0 = 8;  // warps 8-11: correction and epilogue owners
constexpr int kLoadWarpF = 12;
constexpr int kQkWarpF = 13;   // also allocates and frees the tensor memory
constexpr int kPvWarpF = 14;
constexpr int kGroupF = 128;
constexpr int kStagesF = 3;
constexpr uint32_t kTmemColsF = 512;
constexpr uint32_t kColSF = 0;     // two int32 score buffers of 128 columns; P overlays them
constexpr uint32_t kColOF = 256;   // the FP32 output accumulator (D columns)
constexpr float kRescaleLog2 = 8.0f;

template <int D>
struct F32Smem {
  alignas(1024) uint8_t q[kQTile * D];
  alignas(1024) uint8_t k[kStagesF][kGroupF * D];
  alignas(1024) uint8_t v[kStagesF][D * kGroupF];
  float r_ring[2][kQTile];
  float m_x[2][kQTile];
  float m_fin[2][kQTile], d_fin[2][kQTile];
  float rcp[kQTile];
  uint8_t corr[2][4];      // per tile parity and quadrant: the accumulator rows need rescaling
  uint64_t q_full;
  uint64_t kv_full[kStagesF], kv_empty[kStagesF];
  uint64_t s_full[2], s_free[2];
  uint64_t p_full[2], r_free[2];
  uint64_t o_acc[4];       // o_acc[t & 3] completes when the PV MMAs of tile t are done
  uint64_t c_done;         // completes once per rescaled tile when the accumulator is scaled
  uint64_t m_full[4][2];
  uint64_t fin, done;
  uint64_t drain_qk, drain_pv;
  uint32_t tmem_base;
  int abort_flag;
};

template <int D>
__device__ __forceinline__ F32Smem<D>& f32_smem() {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  return *reinterpret_cast<F32Smem<D>*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
}

// 32 lanes x 64 columns of 32 bits from registers.
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const uint32_t (&r)[64]) {
#pragma unroll
  for (int c = 0; c < 64; c += 16) tmem_st16(taddr + c, *reinterpret_cast<const uint32_t(*)[16]>(&r[c]));
}

// DBG: the score export of sage_debug_qk_s32, as in the exact mainloop (a
// one-CTA launch for p.dbg_qt/dbg_h/dbg_b that copies the int32 scores of key
// tile p.dbg_tile to p.dbg_out and stores no output).
template <int D, bool DBG>
__global__ void __launch_bounds__(kThreadsF, 1)
    attn_tc_f32_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const AttnParams p) {
  F32Smem<D>& sm = f32_smem<D>();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qt = DBG ? p.dbg_qt : (int)blockIdx.x;
  const int h = DBG ? p.dbg_h : (int)blockIdx.y;
  const int b = DBG ? p.dbg_b : (int)blockIdx.z;
  const int bh = b * p.H + h;
  const int T = p.T64;
  const int G = (T + 1) >> 1;
  volatile int* abort_flag = &sm.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kStagesF; ++s) {
      mbar_init(&sm.kv_full[s], 1);
      mbar_init(&sm.kv_empty[s], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.s_full[i], 1);
      mbar_init(&sm.s_free[i], 1);
      mbar_init(&sm.p_full[i], kQTile);
      mbar_init(&sm.r_free[i], kQTile + 1);  // correction owners and the PV issuer
      for (int q = 0; q < 4; ++q) mbar_init(&sm.m_full[q][i], 32);
    }
    for (int j = 0; j < 4; ++j) mbar_init(&sm.o_acc[j], 1);
    mbar_init(&sm.c_done, kQTile);
    mbar_init(&sm.fin, 2 * kQTile);
    mbar_init(&sm.done, kQTile);
    mbar_init(&sm.drain_qk, 1);
    mbar_init(&sm.drain_pv, 1);
    sm.abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == kQkWarpF) tmem_alloc(&sm.tmem_base, kTmemColsF);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp < kCorrWarp0) {
    // ------------------------------------------------ QK / softmax owners
    const int quad = warp & 3, par = warp >> 2;
    const int i = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16);
    const int row = qt * kQTile + i;
    const int grp = row / kQGroup;
    const float qs = grp < p.G32 ? p.q_scale[(size_t)bh * p.G32 + grp] : 0.0f;
    const float* ksc = p.k_scale + (size_t)bh * T;
    const int ntail = p.N - (T - 1) * kKTile;
    float m_own = -INFINITY, d_own = 0.0f;  // this warp's latest used max and partial denominator
    float ks_next = par < T ? ksc[par] : 0.0f;
    auto tile_step = [&](auto tail_tag, int t) -> bool {
      constexpr bool TAIL = decltype(tail_tag)::value;
      const int g = t >> 1, sb = g & 1;
      const uint32_t cols = kColSF + 128 * sb + 64 * par;
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
      const bool m_ready = t == 0 || __all_sync(0xffffffffu, mbar_try(&sm.m_full[quad][par ^ 1], (uint32_t)(((t - 1) >> 1) & 1)));
      const bool r_ready = __all_sync(0xffffffffu, mbar_try(&sm.r_free[par], (uint32_t)(((t >> 1) & 1) ^ 1)));
      const float cs = __fmul_rn(__fmul_rn(qs, ks), p.sl2);
      const float tmax = tile_max<TAIL>(S, cs, ntail);
      // used max: raised to the tile max only when that exceeds it by more
      // than kRescaleLog2, so every p = 2^(s - m) stays <= 2^kRescaleLog2
      float m_prev = -INFINITY;
      if (t > 0) {
        if (!m_ready && !wait_bounded(&sm.m_full[quad][par ^ 1], (uint32_t)(((t - 1) >> 1) & 1), abort_flag,
                                      p.status, 15, p.wait_limit))
          return false;
        m_prev = sm.m_x[par ^ 1][i];
      }
      const float m_new = tmax > m_prev + kRescaleLog2 ? tmax : m_prev;
      sm.m_x[par][i] = m_new;
      mbar_arrive(&sm.m_full[quad][par]);
      // the accumulator is empty before tile 0, so nothing is rescaled there
      const float r = (t == 0 || m_new == m_prev) ? 1.0f : ex2(__fsub_rn(m_prev, m_new));
      uint32_t P[16];
      const float rs = tile_exp<TAIL>(lane_addr + cols, cs, m_new, ntail, P);
      d_own = (m_own == m_new) ? __fadd_rn(d_own, rs) : __fadd_rn(__fmul_rn(d_own, ex2(__fsub_rn(m_own, m_new))), rs);
      m_own = m_new;
      tmem_st16(lane_addr + cols, P);
      tmem_wait_st();
      const bool need = __any_sync(0xffffffffu, r != 1.0f);
      if (!r_ready &&
          !wait_bounded(&sm.r_free[par], (uint32_t)(((t >> 1) & 1) ^ 1), abort_flag, p.status, 2, p.wait_limit))
        return false;
      sm.r_ring[par][i] = r;
      if (lane == 0) sm.corr[par][quad] = need ? 1 : 0;
      tc_fence_before();
      mbar_arrive(&sm.p_full[par]);
      return true;
    };
    // one copy of the tile code in the loop; a ragged last tile is peeled off
    const int t_full = ntail == kKTile ? T : T - 1;
    bool ok = true;
    int t = par;
    for (; ok && t < t_full; t += 2) ok = tile_step(std::false_type{}, t);
    if (ok && t == T - 1 && t_full < T) tile_step(std::true_type{}, t);
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
  } else if (warp < kLoadWarpF) {
    // ------------------------------------- correction and epilogue owners
    const int quad = warp & 3;
    const int i = quad * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quad * 32) << 16) + kColOF;
    bool ok = true;
    for (int t = 0; t < T && ok; ++t) {
      const int bi = t & 1;
      // this tile's probabilities first (the wait that usually sleeps), then
      // PV(t - 1), after which the accumulator holds tiles 0 .. t-1.  The
      // o_acc parity is unambiguous: this warp saw tile t - 5 complete on the same
      // barrier, and the next MMAs that complete it, PV(t + 3), need the
      // probabilities of tile t + 3, which wait for this warp's r_free
      // arrival for tile t + 1.
      if (!wait_bounded(&sm.p_full[bi], (uint32_t)((t >> 1) & 1), abort_flag, p.status, 3, p.wait_limit)) break;
      if (t > 0 && !wait_bounded(&sm.o_acc[(t - 1) & 3], (uint32_t)(((t - 1) >> 2) & 1), abort_flag, p.status, 20,
                                 p.wait_limit))
        break;
      // r and the flags are read before the arrival: after it the softmax
      // owners of tile t + 2 may overwrite them
      const float r = sm.r_ring[bi][i];
      const uint32_t flags = *reinterpret_cast<volatile uint32_t*>(&sm.corr[bi][0]);
      mbar_arrive(&sm.r_free[bi]);
      if (flags == 0) continue;
      // every quadrant takes part, so c_done completes once per rescaled tile
      if ((flags >> (8 * quad)) & 0xFFu) {
        tc_fence_after();
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 64) {
          uint32_t o[64];
          tmem_ld64(lane_addr + c0, o);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 64; ++c) o[c] = __float_as_uint(__fmul_rn(__uint_as_float(o[c]), r));
          tmem_st64(lane_addr + c0, o);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&sm.c_done);
    }
    // epilogue: the last PV MMAs have completed and 1/d is known
    if (!DBG && ok && T > 0 &&
        wait_bounded(&sm.o_acc[(T - 1) & 3], (uint32_t)(((T - 1) >> 2) & 1), abort_flag, p.status, 21, p.wait_limit) &&
        wait_bounded(&sm.done, 0, abort_flag, p.status, 5, p.wait_limit) && !*abort_flag) {
      tc_fence_after();
      const int row = qt * kQTile + i;
      const float rc = sm.rcp[i];
      const float* vs = p.v_scale + (size_t)bh * D;
      uint16_t* dst = p.out + b * p.os_b + (int64_t)row * p.os_n + h * p.os_h;
#pragma unroll
      for (int c0 = 0; c0 < D; c0 += 64) {
        uint32_t o[64];
        tmem_ld64(lane_addr + c0, o);
        tmem_wait_ld();
        if (row < p.N) {
#pragma unroll
          for (int c = 0; c < 64; c += 8) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int cc = c0 + c + 2 * e;
              const uint32_t lo = f32_to_bf16_rn(__fmul_rn(__fmul_rn(__uint_as_float(o[c + 2 * e]), rc), vs[cc]));
              const uint32_t hi =
                  f32_to_bf16_rn(__fmul_rn(__fmul_rn(__uint_as_float(o[c + 2 * e + 1]), rc), vs[cc + 1]));
              w[e] = lo | (hi << 16);
            }
            *reinterpret_cast<uint4*>(dst + c0 + c) = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
      }
    }
  } else if (warp == kLoadWarpF) {
    // ------------------------------------------------------------ producer
    const bool leader = lane == 0;
    int issued = 0;
    if (leader) {
      mbar_expect_tx(&sm.q_full, kQTile * D);
      tma_load_3d(sm.q, &tm_q, 0, qt * kQTile, bh, &sm.q_full);
    }
    for (int g = 0; g < G; ++g) {
      const int st = g % kStagesF;
      const bool ok =
          wait_bounded(&sm.kv_empty[st], (uint32_t)(((g / kStagesF) & 1) ^ 1), abort_flag, p.status, 6, p.wait_limit);
      __syncwarp();
      if (!ok) break;
      if (p.stall_tile >= 0 && p.stall_tile / 2 == g) continue;  // test hook: this stage never arrives
      if (leader) {
        mbar_expect_tx(&sm.kv_full[st], 2 * kGroupF * D);
        tma_load_3d(sm.k[st], &tm_k, 0, g * kGroupF, bh, &sm.kv_full[st]);
        tma_load_3d(sm.v[st], &tm_v, g * kGroupF, 0, bh, &sm.kv_full[st]);
      }
      issued = g + 1;
    }
    wait_bounded(&sm.q_full, 0, abort_flag, nullptr, 7, p.wait_limit, false);
    for (int u = max(0, issued - kStagesF); u < issued; ++u)
      if (!(p.stall_tile >= 0 && p.stall_tile / 2 == u))
        wait_bounded(&sm.kv_full[u % kStagesF], (uint32_t)((u / kStagesF) & 1), abort_flag, nullptr, 8,
                     p.wait_limit, false);
  } else if (warp == kQkWarpF) {
    // ----------------------------------------------------------- QK issuer
    const bool leader = lane == 0;
    const uint32_t iqk = idesc_qk(kGroupF);
    const uint64_t qdesc = smem_desc(sm.q, D);
    bool ok = wait_bounded(&sm.q_full, 0, abort_flag, p.status, 9, p.wait_limit);
    __syncwarp();
    for (int g = 0; ok && g < G; ++g) {
      const int st = g % kStagesF, sb = g & 1;
      ok = wait_bounded(&sm.s_free[sb], (uint32_t)(((g >> 1) & 1) ^ 1), abort_flag, p.status, 11, p.wait_limit) &&
           wait_bounded(&sm.kv_full[st], (uint32_t)((g / kStagesF) & 1), abort_flag, p.status, 10, p.wait_limit);
      __syncwarp();
      if (!ok) break;
      tc_fence_after();
      if (leader) {
        const uint64_t kdesc = smem_desc(sm.k[st], D);
#pragma unroll
        for (int kk = 0; kk < D / 32; ++kk)
          mma_i8_ss(tmem + kColSF + 128 * sb, qdesc + 2 * kk, kdesc + 2 * kk, iqk, kk > 0);
        tc_commit(&sm.s_full[sb]);
      }
    }
    __syncwarp();
    if (leader) tc_commit(&sm.drain_qk);
    __syncwarp();
    wait_bounded(&sm.drain_qk, 0, abort_flag, nullptr, 14, p.wait_limit, false);
  } else if (warp == kPvWarpF) {
    // ----------------------------------------------------------- PV issuer
    const bool leader = lane == 0;
    const uint32_t ipv = idesc_pv_f32<D>();
    int ncorr = 0;
    for (int t = 0; t < T; ++t) {
      const int g = t >> 1, sb = g & 1, st = g % kStagesF, half = t & 1;
      bool ok = wait_bounded(&sm.p_full[half], (uint32_t)((t >> 1) & 1), abort_flag, p.status, 12, p.wait_limit) &&
                (half == 1 ||
                 wait_bounded(&sm.kv_full[st], (uint32_t)((g / kStagesF) & 1), abort_flag, p.status, 18, p.wait_limit));
      __syncwarp();
      if (!ok) break;
      // a rescaled tile waits until the correction owners have scaled the
      // accumulator; lane 0's reading of the flags decides for the warp
      const uint32_t flags = __shfl_sync(0xffffffffu, *reinterpret_cast<volatile uint32_t*>(&sm.corr[half][0]), 0);
      if (flags != 0) {
        ok = wait_bounded(&sm.c_done, (uint32_t)(ncorr & 1), abort_flag, p.status, 19, p.wait_limit);
        __syncwarp();
        if (!ok) break;
        ++ncorr;
      }
      tc_fence_after();
      if (leader) {
        mbar_arrive(&sm.r_free[half]);  // seen: p_full of this parity may complete again
        const uint64_t vdesc = smem_desc(sm.v[st], kGroupF) + 4 * half;
#pragma unroll
        for (int sl = 0; sl < 2; ++sl)
          mma_f8_ts(tmem + kColOF, tmem + kColSF + 128 * sb + 64 * half + 8 * sl, vdesc + 2 * sl, ipv,
                    (t > 0 || sl > 0) ? 1u : 0u);
        tc_commit(&sm.o_acc[t & 3]);
        if (half == 1 || t + 1 == T) {
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
  if (warp == kQkWarpF) tmem_free(tmem, kTmemColsF);
}

template <int D>
size_t f32_smem_bytes() {
  const size_t need = sizeof(F32Smem<D>) + 1024;
  return need > 120 * 1024 ? need : 120 * 1024;  // one CTA (and one 512-column TMEM request) per SM
}

template <int D, bool DBG>
int launch_f32(const AttnParams& p, cudaStream_t s) {
  CUtensorMap mq, mk, mv;
  const uint64_t bh = (uint64_t)p.B * p.H;
  if (!make_map(&mq, p.q8, D, p.Nq, bh, D, (uint64_t)p.Nq * D, D, kQTile) ||
      !make_map(&mk, p.k8, D, p.Nk, bh, D, (uint64_t)p.Nk * D, D, kGroupF) ||
      !make_map(&mv, p.v8, p.Nk, D, bh, p.Nk, (uint64_t)D * p.Nk, kGroupF, D))
    return SAGE_ERR_CUDA;
  auto* fn = attn_tc_f32_kernel<D, DBG>;
  const size_t smem = f32_smem_bytes<D>();
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return SAGE_ERR_CUDA;
  const dim3 grid = DBG ? dim3(1, 1, 1) : dim3(p.Nq / kQTile, p.H, p.B);
  fn<<<grid, kThreadsF, smem, s>>>(mq, mk, mv, p);
  return cudaGetLastError() == cudaSuccess ? SAGE_OK : SAGE_ERR_CUDA;
}

}  // namespace

int launch_attn_tc_f32(const AttnParams& p, cudaStream_t s) {
  if (p.D == 128) return p.dbg_out ? launch_f32<128, true>(p, s) : launch_f32<128, false>(p, s);
  if (p.D == 64) return p.dbg_out ? launch_f32<64, true>(p, s) : launch_f32<64, false>(p, s);
  return SAGE_ERR_UNSUPPORTED;
}

}  // namespace sage
