// INT8 code generation shared by the prepass kernels.
//
// The code of x with inverse scale inv is RNE(fl32(x * inv)) clamped to
// [-127, 127] ("Sage2 Blackwell Mainloop", section "Existing Contract":
// symmetric INT8 with an FP32 scale per 32-row Q group and per 64-row K
// block).  Two forms give the same bytes:
//   - the reference form: float-to-int conversion and the clamp, valid for
//     every input (NaN converts to 0, +-inf to the clamp bounds);
//   - the fast form, for a group whose amax (>= every |x|, NaN-propagating)
//     and inv = fl32(127 / amax) are finite.  Then |x * inv| <= 127 (1 +
//     2^-24) and |fl32(x * inv)| < 127.5, so the clamp never acts.  Adding
//     1.5 * 2^23 rounds to an integer: in [2^23, 2^24) FP32 values are
//     spaced 1 apart, and 1.5 * 2^23 is even, so ties still go to even.
//     fl32(y + 1.5 * 2^23) is therefore exactly 1.5 * 2^23 + RNE(y), and the
//     low byte of its bits is RNE(y) as a two's complement byte.
#pragma once
#include "sage_common.cuh"

namespace sage {

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Reference form of one code.
__device__ __forceinline__ uint32_t i8_code(float x, float inv) {
  int r = __float2int_rn(__fmul_rn(x, inv));
  r = max(-127, min(127, r));
  return static_cast<uint32_t>(r) & 0xFFu;
}

__device__ __forceinline__ uint2 i8_codes8_ref(const float (&x)[8], float inv) {
  uint2 o;
  o.x = i8_code(x[0], inv) | i8_code(x[1], inv) << 8 | i8_code(x[2], inv) << 16 | i8_code(x[3], inv) << 24;
  o.y = i8_code(x[4], inv) | i8_code(x[5], inv) << 8 | i8_code(x[6], inv) << 16 | i8_code(x[7], inv) << 24;
  return o;
}

constexpr float kRoundMagic = 12582912.0f;  // 1.5 * 2^23

// Low bytes of four words, in order, in one word.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t b0, uint32_t b1, uint32_t b2, uint32_t b3) {
  return __byte_perm(__byte_perm(b0, b1, 0x0040), __byte_perm(b2, b3, 0x0040), 0x5410);
}

// Fast form of eight codes (see above for when it applies).
__device__ __forceinline__ uint2 i8_codes8_fast(const float (&x)[8], float inv) {
  uint32_t b[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) b[j] = __float_as_uint(__fadd_rn(__fmul_rn(x[j], inv), kRoundMagic));
  return make_uint2(low_bytes4(b[0], b[1], b[2], b[3]), low_bytes4(b[4], b[5], b[6], b[7]));
}

// max that returns NaN when either operand is NaN.
__device__ __forceinline__ float fmax_nan(float a, float b) {
  float d;
  asm("max.NaN.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// The largest BF16 magnitude among eight packed values, as bits (NaN and
// inf are larger than every finite magnitude).
__device__ __forceinline__ uint32_t amax_bits8(const uint4& u, uint32_t m) {
  m = max_u16x2(m, u.x & 0x7FFF7FFFu);
  m = max_u16x2(m, u.y & 0x7FFF7FFFu);
  m = max_u16x2(m, u.z & 0x7FFF7FFFu);
  return max_u16x2(m, u.w & 0x7FFF7FFFu);
}

__device__ __forceinline__ uint32_t halves_max(uint32_t m) { return max(m & 0xFFFFu, m >> 16); }

// True when a group with this (NaN-propagating) amax takes the fast form.
__device__ __forceinline__ bool codes_fast(float amax, float inv) {
  return amax <= 3.4028235e38f && inv <= 3.4028235e38f;  // false for NaN and inf
}

// ------------------------------------------------------------- K mean
// The K mean is the FP64 sum of the FP64 chunk partials in chunk order,
// divided by N in FP64 and rounded once to FP32.  A nonzero partial p is a
// multiple of 2^lo(p), its lowest set bit, and below 2^(hi(p)+1) in
// magnitude.  With lo and hi the minimum and maximum over a channel's
// chunks, every sum of partials is a multiple of 2^lo below
// 2^(ceil(log2 T64) + hi + 1): exact in FP64 when
// ceil(log2 T64) + hi - lo <= 52, and then any order of the additions gives
// the chunk-order sum bit for bit.
constexpr int kExpBias = 1100;  // keeps kExpBias + hi and kExpBias - lo positive

__device__ __forceinline__ void partial_bits(double p, int& hi, int& lo) {
  // p is a nonzero sum of BF16 values: a normal FP64 number
  const unsigned long long bits = (unsigned long long)__double_as_longlong(p);
  const int e = (int)((bits >> 52) & 0x7FFu);
  const unsigned long long sig = (bits & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  hi = e - 1023;
  lo = e - 1075 + __ffsll((long long)sig) - 1;
}

__device__ __forceinline__ bool partials_exact(int log2t, int hi, int lo) { return log2t + hi - lo <= 52; }

}  // namespace sage
