/*
 * CPU oracle for SageAttention-2-style quantized non-causal attention
 * (INT8 QK^T, FP8-E4M3 PV with an FP16 per-K32 "instantaneous buffer",
 * FP32 online softmax).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow, single-threaded
 * statement of what the GPU path computes.  Only the tests, the smoke check
 * and the benchmark's CPU-baseline leg may load it; the product path never
 * does.  It shares no code with the CUDA library.
 *
 * Sources (the research pages this method is described on):
 *  - "Sage2 Blackwell Mainloop", section "Existing Contract":
 *    projection-strided BF16 NHD input, per-warp INT8 Q in 128-row blocks of
 *    32-row warp groups, per-block INT8 K with 64-row blocks, FP8 V with a
 *    per-channel scale, fp32+fp16 instantaneous-buffer accumulation,
 *    contiguous BF16 NHD output.
 *  - "State-Ownership Architecture Decision", section "Non-Negotiable
 *    Dataflow": exact global K mean and V scale prepasses; all K64/V64 tiles
 *    in increasing order; per tile QK,
 *    score scaling, max update, denominator update, FP8 probability
 *    conversion, two K32 FP16 PV MMAs and the FP32 RO addition; and the
 *    "exact handoff record" paragraph: ro_rescale (the old-max rescale) is
 *    applied before the tile's PV, and the final normalisation uses the FP32
 *    reciprocal of d, then the V scale, then BF16 conversion.
 *  - "Sage2 SM89 Temporal Pair Experiment", section "Candidate": the
 *    per-tile order QK -> update_mdo -> accumulate_d -> RS_32_to_8 -> PV.
 *
 * Readings taken where the pages are silent:
 *  R1 K mean: per (b,h,d) an FP64 sum over tokens, sequential inside each
 *     64-token chunk, then the chunk partials added sequentially in chunk
 *     order; km = float(sum / N), one round-to-nearest-even.
 *  R2 Q/K quantisation: symmetric, no zero point, range +-127:
 *     amax = max |x| over the group (32 consecutive Q rows, 64 consecutive K
 *     rows, all D channels; the last group is ragged); scale = amax/127 and
 *     inv = 127/amax (both correctly rounded FP32 divisions); byte =
 *     clamp(rint_even(fl32(x*inv)), -127, 127); amax == 0 -> scale 0, bytes 0.
 *     K is smoothed first: x' = fl32(x - km[d]).  Q is quantised raw (the
 *     softmax scale is not folded into Q).
 *  R3 V quantisation: per (b,h,d) amax over all N tokens; scale = amax/448,
 *     inv = 448/amax; byte = E4M3(fl32(x*inv)) with OCP E4M3 "FN" encoding
 *     (bias 7, max 448, no infinities), round-to-nearest-even, saturating;
 *     a value that rounds to zero keeps its sign (0x80 for negatives).
 *  R4 Score scale: sl2 = fl32(double(sm_scale) * log2(e)); sm_scale <= 0
 *     means fl32(1/sqrt(D)); per (32-row Q group g, 64-key tile t):
 *     c = fl32(fl32(q_scale[g]*k_scale[t]) * sl2); s = fl32(float(S)*c).
 *     Keys j >= N of the last tile are masked (s = -inf).
 *  R5 Exponentials are base 2 (scores carry log2(e)); the oracle evaluates
 *     exp2 in double and rounds to float.
 *  R6 The denominator takes the FP32 probabilities before FP8 conversion:
 *     d = fl32(fl32(d*r) + rowsum), rowsum summed in key order in FP32.
 *  R7 PV: each K32 slice (keys 0-31, then 32-63 of the tile) is one FP16
 *     instantaneous buffer: tmp = fp16_rne(exact sum of p8*v8), then
 *     RO = fl32(RO + float(tmp)) per slice, in slice order.
 *  R8 Output: rcp = fl32(1/d); out = bf16_rne(fl32(fl32(RO*rcp)*v_scale[d])).
 *  R11 Q/K producer (RMSNorm + split-half RoPE before the Q/K quantisation;
 *     "Sage2 Blackwell Mainloop", section "Completed P1 And P2", names the
 *     fused producer but gives no formula or rounding).  Per (b, n, h) row x
 *     of D BF16 values, BF16 weight w[D], FP32 tables cos/sin[N][D/2]:
 *       ss = FP32 sum of fl32(x_d*x_d) in channel order;
 *       r  = fl32(1 / fl32(sqrt(fl32(fl32(ss/D) + eps))))   (correctly rounded);
 *       y_d = bf16(fl32(bf16(fl32(x_d*r)) * w_d));
 *       for j < D/2, a = y_j, b = y_{j+D/2}, c = cos[n][j], s = sin[n][j]:
 *         z_j       = bf16(fl32(fl32(a*c) - fl32(b*s))),
 *         z_{j+D/2} = bf16(fl32(fl32(b*c) + fl32(a*s))).
 *     z then goes through R1/R2 exactly as the raw Q and K do.
 *
 * Build: gcc -O2 -ffp-contract=off (no -ffast-math).  Defining
 * ORACLE_PLANT=<n> builds a deliberately wrong variant, used only by the
 * tests that show the pins catch such mistakes.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifndef ORACLE_PLANT
#define ORACLE_PLANT 0
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL 1
#define ORACLE_ENOMEM 2

/* ---------------------------------------------------------------- formats */

static float f32_from_bits(uint32_t u) { float f; memcpy(&f, &u, 4); return f; }
static uint32_t bits_from_f32(float f) { uint32_t u; memcpy(&u, &f, 4); return u; }

/* BF16 -> FP32 is exact: the BF16 bits are the high half of the FP32 bits. */
static float bf16_to_f32(uint16_t h) { return f32_from_bits((uint32_t)h << 16); }

/* FP32 -> BF16, round to nearest, ties to even; NaN stays NaN. */
static uint16_t f32_to_bf16(float x) {
  uint32_t u = bits_from_f32(x);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* Decode one OCP E4M3 (FN) byte: bias 7; exponent field 0 is subnormal
 * (m/8 * 2^-6); S.1111.111 is NaN; no infinities. */
static double e4m3_decode(uint8_t b) {
  int sign = b >> 7, e = (b >> 3) & 15, m = b & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0) v = ldexp((double)m, -9);           /* m/8 * 2^-6 */
  else v = ldexp(1.0 + m / 8.0, e - 7);
  return sign ? -v : v;
}

/* FP32 -> E4M3, round to nearest even, saturate to +-448, NaN -> 0x7F.
 * Written from the format: the representable magnitudes are k * 2^(E-3)
 * for the binade [2^E, 2^(E+1)), E >= -6, and k * 2^-9 below 2^-6. */
static uint8_t e4m3_encode(float xf) {
  double x = (double)xf;
  if (isnan(x)) return 0x7F;
  uint8_t sign = signbit(x) ? 0x80 : 0x00;
  double a = fabs(x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  /* quantum of the binade that holds a (subnormal range below 2^-6) */
  int E;
  if (a < ldexp(1.0, -6)) E = -6;
  else { frexp(a, &E); E -= 1; }                  /* a in [2^E, 2^(E+1)) */
  double q = ldexp(1.0, E - 3);
  double k = a / q;                               /* exact: power-of-two division */
  double kr = nearbyint(k);                       /* default rounding: ties to even */
  double r = kr * q;
  if (r > 448.0) r = 448.0;                       /* cannot happen below 448, kept for clarity */
  if (r == 0.0) return sign;
  /* encode r exactly */
  int e2;
  frexp(r, &e2); e2 -= 1;                         /* r in [2^e2, 2^(e2+1)) */
  uint8_t code;
  if (e2 < -6) {                                  /* subnormal: r = m * 2^-9 */
    code = (uint8_t)(r / ldexp(1.0, -9));
  } else {
    int mant = (int)((r / ldexp(1.0, e2) - 1.0) * 8.0);
    code = (uint8_t)(((e2 + 7) << 3) | mant);
  }
  return (uint8_t)(sign | code);
}

/* double -> IEEE binary16, one rounding, to nearest even; overflow to inf. */
static uint16_t f64_to_f16(double x) {
  if (isnan(x)) return 0x7E00;
  uint16_t sign = signbit(x) ? 0x8000 : 0;
  double a = fabs(x);
  if (a == 0.0) return sign;
  int E;
  frexp(a, &E); E -= 1;                           /* a in [2^E, 2^(E+1)) */
  if (E < -14) E = -14;                           /* subnormal quantum 2^-24 */
  double q = ldexp(1.0, E - 10);
  double r = nearbyint(a / q) * q;
  if (r == 0.0) return sign;
  if (r > 65504.0) return (uint16_t)(sign | 0x7C00);
  int e2;
  frexp(r, &e2); e2 -= 1;
  if (e2 < -14) return (uint16_t)(sign | (uint16_t)(r / ldexp(1.0, -24)));
  uint16_t mant = (uint16_t)((r / ldexp(1.0, e2) - 1.0) * 1024.0);
  return (uint16_t)(sign | (uint16_t)((e2 + 15) << 10) | mant);
}

static float f16_to_f32(uint16_t h) {
  int sign = h >> 15, e = (h >> 10) & 31, m = h & 1023;
  double v;
  if (e == 31) v = m ? NAN : INFINITY;
  else if (e == 0) v = ldexp((double)m, -24);
  else v = ldexp(1.0 + m / 1024.0, e - 15);
  return (float)(sign ? -v : v);
}

/* round-half-even to integer, then clamp to the INT8 code range */
static int8_t quant_i8(float prod) {
#if ORACLE_PLANT == 14
  float r = roundf(prod); /* planted: ties away from zero */
#else
  float r = nearbyintf(prod);
#endif
  if (r > 127.0f) r = 127.0f;
  if (r < -127.0f) r = -127.0f;
  return (int8_t)r;
}

/* Exported format helpers (the pin tests compare them with library
 * conversions). */
uint8_t oracle_e4m3_encode(float x) { return e4m3_encode(x); }
double oracle_e4m3_decode(uint8_t b) { return e4m3_decode(b); }
uint16_t oracle_f16_round(double x) { return f64_to_f16(x); }
float oracle_f16_decode(uint16_t h) { return f16_to_f32(h); }
uint16_t oracle_bf16_round(float x) { return f32_to_bf16(x); }

/* --------------------------------------------------------------- geometry */

static int check_dims(int B, int N, int H, int D) {
  return (B < 0 || N < 0 || H < 0 || D <= 0 || D > 256) ? ORACLE_EINVAL : ORACLE_OK;
}
#define IDX_IN(b, n, h) ((int64_t)(b) * sb + (int64_t)(n) * sn + (int64_t)(h) * sh)

/* ------------------------------------------------------------ a1: K mean
 * Reading R1.  km[b][h][d]. */
int oracle_k_mean(const uint16_t* k, int64_t sb, int64_t sn, int64_t sh,
                  int B, int N, int H, int D, float* km) {
  if (check_dims(B, N, H, D)) return ORACLE_EINVAL;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int d = 0; d < D; ++d) {
#if ORACLE_PLANT == 19
        float total = 0.0f; /* planted: the sums kept in FP32 */
#else
        double total = 0.0;
#endif
        for (int c0 = 0; c0 < N; c0 += 64) {
#if ORACLE_PLANT == 19
          float part = 0.0f;
          int c1 = c0 + 64 < N ? c0 + 64 : N;
          for (int n = c0; n < c1; ++n) part += bf16_to_f32(k[IDX_IN(b, n, h) + d]);
#else
          double part = 0.0;
          int c1 = c0 + 64 < N ? c0 + 64 : N;
          for (int n = c0; n < c1; ++n) part += (double)bf16_to_f32(k[IDX_IN(b, n, h) + d]);
#endif
          total += part;
        }
#if ORACLE_PLANT == 1
        km[((int64_t)b * H + h) * D + d] = 0.0f; /* planted: smoothing dropped */
#elif ORACLE_PLANT == 15
        km[((int64_t)b * H + h) * D + d] =      /* planted: mean over the padded length */
            N > 0 ? (float)(total / (double)(64 * ((N + 63) / 64))) : 0.0f;
#else
        km[((int64_t)b * H + h) * D + d] = N > 0 ? (float)(total / (double)N) : 0.0f;
#endif
      }
  return ORACLE_OK;
}

/* shared rule of R2 for one group of rows [r0, r1) of one (b, h):
 * x'(n, d) = fl32(bf16(n, d) - sub[d]) (sub may be NULL). */
static void quant_group_i8(const uint16_t* x, int64_t sb, int64_t sn, int64_t sh, int b, int h,
                           int r0, int r1, int D, const float* sub, int8_t* out_rows /*[r1-r0][D]*/,
                           float* scale_out) {
  float amax = 0.0f;
  for (int n = r0; n < r1; ++n)
    for (int d = 0; d < D; ++d) {
      float v = bf16_to_f32(x[IDX_IN(b, n, h) + d]);
      if (sub) v = v - sub[d];
      float a = fabsf(v);
      if (a > amax) amax = a;
    }
  if (amax == 0.0f) {
    *scale_out = 0.0f;
    memset(out_rows, 0, (size_t)(r1 - r0) * D);
    return;
  }
#if ORACLE_PLANT == 2
  float scale = 127.0f / amax, inv = amax / 127.0f; /* planted: scale inverted */
#else
  float scale = amax / 127.0f, inv = 127.0f / amax;
#endif
  *scale_out = scale;
  for (int n = r0; n < r1; ++n)
    for (int d = 0; d < D; ++d) {
      float v = bf16_to_f32(x[IDX_IN(b, n, h) + d]);
      if (sub) v = v - sub[d];
      out_rows[(int64_t)(n - r0) * D + d] = quant_i8(v * inv);
    }
}

/* ----------------------------------------------------------- a2: Q quant
 * q8[b][h][n][d] (logical, unpadded), q_scale[b][h][ceil(N/32)]. */
int oracle_quant_q(const uint16_t* q, int64_t sb, int64_t sn, int64_t sh, int B, int N, int H, int D,
                   int8_t* q8, float* q_scale) {
  if (check_dims(B, N, H, D)) return ORACLE_EINVAL;
#if ORACLE_PLANT == 3
  const int G = 64; /* planted: wrong Q group size */
#else
  const int G = 32;
#endif
  int ng = (N + 31) / 32;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int g0 = 0; g0 < N; g0 += G) {
        int g1 = g0 + G < N ? g0 + G : N;
        float sc;
        quant_group_i8(q, sb, sn, sh, b, h, g0, g1, D, NULL,
                       q8 + (((int64_t)b * H + h) * N + g0) * D, &sc);
        for (int g = g0 / 32; g < (g1 + 31) / 32 && g < ng; ++g)
          q_scale[((int64_t)b * H + h) * ng + g] = sc;
      }
  return ORACLE_OK;
}

/* ----------------------------------------------------------- a3: K quant
 * k8[b][h][n][d] (logical), k_scale[b][h][ceil(N/64)]; km from a1. */
int oracle_quant_k(const uint16_t* k, int64_t sb, int64_t sn, int64_t sh, int B, int N, int H, int D,
                   const float* km, int8_t* k8, float* k_scale) {
  if (check_dims(B, N, H, D)) return ORACLE_EINVAL;
  int nt = (N + 63) / 64;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int t = 0; t < nt; ++t) {
        int r0 = 64 * t, r1 = r0 + 64 < N ? r0 + 64 : N;
        quant_group_i8(k, sb, sn, sh, b, h, r0, r1, D, km + ((int64_t)b * H + h) * D,
                       k8 + (((int64_t)b * H + h) * N + r0) * D,
                       &k_scale[((int64_t)b * H + h) * nt + t]);
      }
  return ORACLE_OK;
}

/* ----------------------------------------- producer: RMSNorm + RoPE (R11)
 * z[b][n][h][d] BF16 bits, contiguous, from the strided view x. */
int oracle_norm_rope(const uint16_t* x, int64_t sb, int64_t sn, int64_t sh, int B, int N, int H, int D,
                     const uint16_t* w, const float* cos_t, const float* sin_t, float eps, uint16_t* z) {
  if (check_dims(B, N, H, D) || (D & 1) || !w || !cos_t || !sin_t || !z) return ORACLE_EINVAL;
  const int half = D / 2;
  float* y = (float*)malloc(sizeof(float) * (size_t)D);
  if (!y) return ORACLE_ENOMEM;
  for (int b = 0; b < B; ++b)
    for (int n = 0; n < N; ++n)
      for (int h = 0; h < H; ++h) {
        const uint16_t* row = x + b * sb + n * sn + h * sh;
        float ss = 0.0f;
        for (int d = 0; d < D; ++d) {
          const float v = bf16_to_f32(row[d]);
          ss = ss + v * v;
        }
        const float mean = ss / (float)D;
        const float r = 1.0f / sqrtf(mean + eps);
        for (int d = 0; d < D; ++d) {
          const float xn = bf16_to_f32(f32_to_bf16(bf16_to_f32(row[d]) * r));
          y[d] = bf16_to_f32(f32_to_bf16(xn * bf16_to_f32(w[d])));
        }
        uint16_t* out = z + (((size_t)b * N + n) * H + h) * D;
        for (int j = 0; j < half; ++j) {
          const float a = y[j], bb = y[j + half];
          const float c = cos_t[(size_t)n * half + j], s = sin_t[(size_t)n * half + j];
#if ORACLE_PLANT == 9
          out[j] = f32_to_bf16(a * c + bb * s);      /* planted: rotation sign */
#else
          out[j] = f32_to_bf16(a * c - bb * s);
#endif
          out[j + half] = f32_to_bf16(bb * c + a * s);
        }
      }
  free(y);
  return ORACLE_OK;
}

/* ----------------------------------------------------------- a4: V quant
 * v8[b][h][n][d] (logical, token-major; the GPU stores it transposed),
 * v_scale[b][h][d]. */
int oracle_quant_v(const uint16_t* v, int64_t sb, int64_t sn, int64_t sh, int B, int N, int H, int D,
                   uint8_t* v8, float* v_scale) {
  if (check_dims(B, N, H, D)) return ORACLE_EINVAL;
  for (int b = 0; b < B; ++b)
    for (int h = 0; h < H; ++h)
      for (int d = 0; d < D; ++d) {
        float amax = 0.0f;
        for (int n = 0; n < N; ++n) {
          float a = fabsf(bf16_to_f32(v[IDX_IN(b, n, h) + d]));
          if (a > amax) amax = a;
        }
        float scale = amax > 0.0f ? amax / 448.0f : 0.0f;
        float inv = amax > 0.0f ? 448.0f / amax : 0.0f;
        v_scale[((int64_t)b * H + h) * D + d] = scale;
        for (int n = 0; n < N; ++n) {
          float x = bf16_to_f32(v[IDX_IN(b, n, h) + d]);
          v8[(((int64_t)b * H + h) * N + n) * D + d] = amax > 0.0f ? e4m3_encode(x * inv) : 0;
        }
      }
  return ORACLE_OK;
}

/* R4: the per-call constant sl2 */
static float score_log2_scale(float sm_scale, int D) {
  if (!(sm_scale > 0.0f)) sm_scale = (float)(1.0 / sqrt((double)D));
#if ORACLE_PLANT == 4
  return sm_scale; /* planted: natural-base scores fed to exp2 */
#else
  return (float)((double)sm_scale * 1.4426950408889634074);
#endif
}

/* --------------------------------------------------- a5..a9: attention rows
 * For one (b, h) and query rows [row0, row0 + rows): out[rows][D] BF16 bits.
 * Inputs are the logical quantised tensors of a2..a4.  stats (optional)
 * receives the final (m, d) per row. */
int oracle_attn_rows(const int8_t* q8, const float* q_scale, const int8_t* k8, const float* k_scale,
                     const uint8_t* v8, const float* v_scale, int B, int N, int H, int D,
                     float sm_scale, int b, int h, int row0, int rows, uint16_t* out, float* stats) {
  if (check_dims(B, N, H, D) || b < 0 || b >= B || h < 0 || h >= H || row0 < 0 || rows < 0 ||
      row0 + rows > N)
    return ORACLE_EINVAL;
  const int ng = (N + 31) / 32, nt = (N + 63) / 64;
  const int64_t bh = (int64_t)b * H + h;
  const int8_t* Q = q8 + bh * N * D;
  const int8_t* K = k8 + bh * N * D;
  const uint8_t* V = v8 + bh * N * D;
  const float sl2 = score_log2_scale(sm_scale, D);
  float* RO = (float*)malloc(sizeof(float) * D);
  double* vdec = (double*)malloc(sizeof(double) * 256);
  if (!RO || !vdec) { free(RO); free(vdec); return ORACLE_ENOMEM; }
  for (int c = 0; c < 256; ++c) vdec[c] = e4m3_decode((uint8_t)c);

  for (int ri = 0; ri < rows; ++ri) {
    const int i = row0 + ri;
#if ORACLE_PLANT == 16
    const float qs = q_scale[bh * ng + i / 64]; /* planted: Q scale read per 64 rows */
#else
    const float qs = q_scale[bh * ng + i / 32];
#endif
    float m = -INFINITY, dsum = 0.0f;
    for (int e = 0; e < D; ++e) RO[e] = 0.0f;

    for (int t = 0; t < nt; ++t) {
      const int j0 = 64 * t, j1 = j0 + 64 < N ? j0 + 64 : N;
      const float c = (qs * k_scale[bh * nt + t]) * sl2;
      float s[64], p[64];
      uint8_t p8[64];
      /* a5 + a6: INT8 QK^T, exact in int32, then the FP32 scale */
      float tmax = -INFINITY;
      for (int jj = 0; jj < 64; ++jj) {
        int j = j0 + jj;
#if ORACLE_PLANT == 13
        if (j >= j1) { s[jj] = 0.0f; continue; }       /* planted: tail keys not masked */
#else
        if (j >= j1) { s[jj] = -INFINITY; continue; }  /* tail mask */
#endif
        int32_t S = 0;
#if ORACLE_PLANT == 5
        for (int e = 0; e < D; ++e) S += (int32_t)Q[(int64_t)i * D + e] * K[(int64_t)j * D + (D - 1 - e)];
#else
        for (int e = 0; e < D; ++e) S += (int32_t)Q[(int64_t)i * D + e] * K[(int64_t)j * D + e];
#endif
        s[jj] = (float)S * c;
        if (s[jj] > tmax) tmax = s[jj];
      }
      /* update_mdo: new max, ro_rescale applied to RO and d */
      const float m_new = m > tmax ? m : tmax;
      const float r = (float)exp2((double)(m - m_new));
#if ORACLE_PLANT != 6 && ORACLE_PLANT != 17 && ORACLE_PLANT != 18
      for (int e = 0; e < D; ++e) RO[e] = RO[e] * r;
#endif
#if ORACLE_PLANT != 6
      dsum = dsum * r;
#endif
      /* accumulate_d on FP32 probabilities, then RS_32_to_8 */
      float rowsum = 0.0f;
      for (int jj = 0; jj < 64; ++jj) {
#if ORACLE_PLANT == 7
        p[jj] = (float)exp2((double)s[jj]); /* planted: max not subtracted */
        (void)m_new;
#else
        p[jj] = (float)exp2((double)(s[jj] - m_new));
#endif
#if ORACLE_PLANT == 10
        rowsum = rowsum + (float)e4m3_decode(e4m3_encode(p[jj])); /* planted: d from E4M3 p */
#else
        rowsum = rowsum + p[jj];
#endif
      }
      dsum = dsum + rowsum;
      for (int jj = 0; jj < 64; ++jj) p8[jj] = e4m3_encode(p[jj]);
      /* PV: two ordered K32 FP16 instantaneous buffers, each added in FP32 */
#if ORACLE_PLANT == 12
      const int SL = 64; /* planted: one K64 FP16 buffer instead of two K32 ones */
#else
      const int SL = 32;
#endif
      for (int sl = 0; sl < 64 / SL; ++sl) {
        for (int e = 0; e < D; ++e) {
          double acc = 0.0;
          for (int jj = SL * sl; jj < SL * sl + SL; ++jj) {
            int j = j0 + jj;
            if (j >= j1) break;
            acc += vdec[p8[jj]] * vdec[V[(int64_t)j * D + e]];
          }
#if ORACLE_PLANT == 11
          RO[e] = RO[e] + (float)acc; /* planted: FP16 buffer rounding skipped */
#else
          RO[e] = RO[e] + f16_to_f32(f64_to_f16(acc));
#endif
        }
      }
#if ORACLE_PLANT == 17
      for (int e = 0; e < D; ++e) RO[e] = RO[e] * r; /* planted: RO rescaled after the tile's PV */
#endif
      m = m_new;
    }
    /* final normalisation: FP32 reciprocal of d, then the V scale, then BF16 */
    const float rcp = 1.0f / dsum;
    for (int e = 0; e < D; ++e) {
#if ORACLE_PLANT == 8
      float o = RO[e] * rcp; /* planted: V scale not applied */
#else
      float o = (RO[e] * rcp) * v_scale[bh * D + e];
#endif
      out[(int64_t)ri * D + e] = f32_to_bf16(o);
    }
    if (stats) { stats[2 * ri] = m; stats[2 * ri + 1] = dsum; }
  }
  free(RO);
  free(vdec);
  return ORACLE_OK;
}

/* int32 QK^T of one (b, h): S[i][j] for rows [row0, row0+rows) and keys
 * [key0, key0+keys); rows/keys beyond N read as zero (the zero padding of
 * the GPU layouts). */
int oracle_qk_s32(const int8_t* q8, const int8_t* k8, int B, int N, int H, int D, int b, int h,
                  int row0, int rows, int key0, int keys, int32_t* S) {
  if (check_dims(B, N, H, D) || b < 0 || b >= B || h < 0 || h >= H || row0 < 0 || key0 < 0 ||
      rows < 0 || keys < 0)
    return ORACLE_EINVAL;
  const int64_t bh = (int64_t)b * H + h;
  for (int ri = 0; ri < rows; ++ri)
    for (int kj = 0; kj < keys; ++kj) {
      int i = row0 + ri, j = key0 + kj;
      int32_t acc = 0;
      if (i < N && j < N)
        for (int e = 0; e < D; ++e)
          acc += (int32_t)q8[(bh * N + i) * D + e] * (int32_t)k8[(bh * N + j) * D + e];
      S[(int64_t)ri * keys + kj] = acc;
    }
  return ORACLE_OK;
}

int oracle_plant(void) { return ORACLE_PLANT; }
