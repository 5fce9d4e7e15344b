// Shared device helpers and launch parameter blocks of the sm_100a library.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "sage_b200.h"

namespace sage {

constexpr int kQTile = 128;   // query rows per Q block (4 groups of 32)
constexpr int kQGroup = 32;   // rows per Q scale
constexpr int kKTile = 64;    // keys per K/V tile and per K scale

__host__ __device__ inline int ceil_div(int a, int b) { return (a + b - 1) / b; }

// Status word at the start of every workspace.
struct DeviceStatus {
  int code;       // SAGE_OK or SAGE_ERR_TIMEOUT / SAGE_ERR_DEVICE
  int where;      // which wait or check gave up
  int block;      // linear block index that flagged it
  int pad;
};

// Everything a mainloop launch needs (device pointers, logical sizes).
struct AttnParams {
  const int8_t* q8;      // [B][H][Nq][D]
  const float* q_scale;  // [B][H][G32]
  const int8_t* k8;      // [B][H][Nk][D]
  const float* k_scale;  // [B][H][T64]
  const uint8_t* v8;     // [B][H][D][Nk]
  const float* v_scale;  // [B][H][D]
  uint16_t* out;         // BF16 [B, N, H, D] strided
  int64_t os_b, os_n, os_h;
  int B, N, H, D;
  int Nq, Nk, G32, T64;
  float sl2;             // fl32(sm_scale * log2 e)
  DeviceStatus* status;
  long long wait_limit;  // clock cycles a bounded device wait may spin
  int stall_tile;        // test hook: the producer withholds this K/V tile (-1: none)
  // score export of the mainloop's own QK path (sage_debug_qk_s32): the CTA
  // of query tile dbg_qt of head (dbg_b, dbg_h) copies the int32 scores of
  // key tile dbg_tile to dbg_out (128 x 64, row-major)
  int dbg_qt, dbg_h, dbg_b, dbg_tile;
  int32_t* dbg_out;
};

constexpr long long kDefaultWaitLimit = 2000000000LL;  // ~1 s at 1.9 GHz

// --------------------------------------------------------------- numerics
// Pack two floats into two E4M3 bytes (round to nearest even, satfinite);
// `lo` lands in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float bf16_bits_to_f32(uint16_t h) {
  return __uint_as_float(((uint32_t)h) << 16);
}

// FP32 -> BF16 with round-to-nearest-even (cvt.rn.bf16.f32).
__device__ __forceinline__ uint16_t f32_to_bf16_rn(float x) {
  uint16_t r;
  asm("cvt.rn.bf16.f32 %0, %1;" : "=h"(r) : "f"(x));
  return r;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// ---------------------------------------------------------------- memory
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_16_zfill(uint32_t dst, const void* src, bool valid) {
  int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// 128-byte swizzle of a byte offset inside a 1024-byte aligned tile: the
// 16-byte chunk index (bits 4..6) is XORed with bits 7..9.  Rows of 64 or
// 128 bytes read through ldmatrix then hit 8 distinct bank groups.
__device__ __forceinline__ uint32_t swz128(uint32_t off) { return off ^ (((off >> 7) & 7u) << 4); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                            uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

}  // namespace sage

// Host-side launchers (defined in the .cu files).
namespace sage {
// Outputs and scratch of the single-launch prepass (device pointers).
struct FusedOut {
  int8_t* q8;
  float* q_scale;
  int8_t* k8;
  float* k_scale;
  float* k_mean;
  uint8_t* v8;
  float* v_scale;
  double* k_part;      // [B][H][T64][D]
  void* sync;          // prepass_sync_bytes(B, H, D), zeroed by the launcher
  DeviceStatus* status;
  long long wait_limit;
  int stall_unit;      // test hook (-1: none)
};
// Inputs of the RMSNorm + RoPE producer (device pointers).
struct NormRopeIn {
  const uint16_t* wq;   // BF16 [D]
  const uint16_t* wk;   // BF16 [D]
  const float* cos_t;   // FP32 [N][D/2]
  const float* sin_t;   // FP32 [N][D/2]
  float eps;
};
int launch_norm_rope_qk(const NormRopeIn& in, const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H,
                        int D, int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean, double* k_part,
                        cudaStream_t s);
void launch_reduce_k_mean(int BH, int N, int D, int T64, const double* k_part, float* k_mean, cudaStream_t s);
// Bytes of the single-launch prepass's zeroed scratch (statistics
// accumulators, counters and flags).
size_t prepass_sync_bytes(int B, int H, int D);
// The single-launch (streaming) prepass, for any shape the separate kernels take.
int launch_prepass_stream(const sage_view_bf16& q, const sage_view_bf16& k, const sage_view_bf16& v, int B, int N,
                          int H, int D, const FusedOut& o, cudaStream_t s);
// Its work list for `grid` CTAs, on the host: (kind, head, tile) triples of
// all n items, and the lag in heads.
int prepass_stream_list(int B, int N, int H, int grid, int* lag, long long n, int* items);
// k_part: B*H*T64*D doubles of scratch; v_amax: B*H*D floats (scratch, cleared by the launch)
int launch_prepass_qk(const sage_view_bf16& q, const sage_view_bf16& k, int B, int N, int H, int D,
                      int8_t* q8, float* q_scale, int8_t* k8, float* k_scale, float* k_mean,
                      double* k_part, cudaStream_t s);
int launch_prepass_v(const sage_view_bf16& v, int B, int N, int H, int D, uint8_t* v8,
                     float* v_scale, float* v_amax, cudaStream_t s);
int launch_attn_mma(const AttnParams& p, cudaStream_t s);
int launch_debug_qk_mma(const AttnParams& p, int b, int h, int q_tile, int k_tile, int32_t* s_out,
                        cudaStream_t s);
int launch_attn_tc(const AttnParams& p, cudaStream_t s);
int launch_attn_tc_f32(const AttnParams& p, cudaStream_t s);
bool tc_available();
}  // namespace sage
