/*
 * Seeded synthetic input generator shared by the CPU oracle's tests, the GPU
 * parity tests and the benchmark.  It holds none of the attention method's
 * arithmetic: it only produces BF16 activations with a stated distribution.
 *
 * Definition (counter based, so any element can be produced independently and
 * the result does not depend on the number of threads):
 *   key(seed, stream)  = mix64(seed * 0xD1B54A32D192ED03 + stream + 1)
 *   word(key, i)       = mix64(key + (i + 1) * 0x9E3779B97F4A7C15)
 *   mix64              = the splitmix64 finaliser (Steele, Lea, Flood,
 *                        "Fast splittable pseudorandom number generators",
 *                        OOPSLA 2014): xor-shift 30, multiply
 *                        0xBF58476D1CE4E5B9, xor-shift 27, multiply
 *                        0x94D049BB133111EB, xor-shift 31.
 *   uniform(key, i)    = ((word >> 11) + 0.5) * 2^-53, in (0, 1)
 *   normal pair p      = Box-Muller on uniform(2p), uniform(2p+1):
 *                        r = sqrt(-2 ln u1); n(2p) = r cos(2 pi u2),
 *                        n(2p+1) = r sin(2 pi u2)            (all in double)
 * An element of a logical [B, N, H, D] tensor with flat index
 * i = ((b*N + n)*H + h)*D + d takes
 *   x = scale * normal(i) + offset[h*D + d]      (offset optional)
 *   x = x * outlier_mult   when uniform(outlier key, i) < outlier_prob
 * and is stored as BF16(float(x)) with round-to-nearest-even.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

static uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static uint64_t stream_key(uint64_t seed, uint32_t stream) {
  return mix64(seed * 0xD1B54A32D192ED03ULL + (uint64_t)stream + 1ULL);
}

static double uniform_at(uint64_t key, uint64_t i) {
  uint64_t w = mix64(key + (i + 1ULL) * 0x9E3779B97F4A7C15ULL);
  return ((double)(w >> 11) + 0.5) * (1.0 / 9007199254740992.0);
}

static double normal_at(uint64_t key, uint64_t i) {
  const double two_pi = 6.283185307179586476925286766559;
  uint64_t p = i >> 1;
  double u1 = uniform_at(key, 2 * p), u2 = uniform_at(key, 2 * p + 1);
  double r = sqrt(-2.0 * log(u1));
  return (i & 1) ? r * sin(two_pi * u2) : r * cos(two_pi * u2);
}

static uint16_t to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

typedef struct {
  uint64_t key, okey;
  int B, N, H, D;
  int64_t sb, sn, sh;
  uint16_t* out;
  float scale;
  const float* offset;
  float oprob, omult;
  int64_t row_begin, row_end; /* rows are (b, n) pairs */
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  for (int64_t row = j->row_begin; row < j->row_end; ++row) {
    int64_t b = row / j->N, n = row % j->N;
    for (int h = 0; h < j->H; ++h) {
      uint16_t* dst = j->out + b * j->sb + n * j->sn + (int64_t)h * j->sh;
      uint64_t base = (uint64_t)((row * j->H + h) * (int64_t)j->D);
      for (int d = 0; d < j->D; ++d) {
        uint64_t i = base + (uint64_t)d;
        double x = (double)j->scale * normal_at(j->key, i);
        if (j->offset) x += (double)j->offset[h * j->D + d];
        if (j->oprob > 0.0f && uniform_at(j->okey, i) < (double)j->oprob) x *= (double)j->omult;
        dst[d] = to_bf16((float)x);
      }
    }
  }
  return 0;
}

/* Fill a strided BF16 view [B, N, H, D] (element strides sb, sn, sh; unit
 * stride over d).  Returns 0 on success, -1 on bad arguments. */
int synth_fill_bf16(uint64_t seed, uint32_t stream, int B, int N, int H, int D,
                    int64_t sb, int64_t sn, int64_t sh, uint16_t* out, float scale,
                    const float* hd_offset, float outlier_prob, float outlier_mult,
                    uint32_t outlier_stream, int nthreads) {
  if (B < 0 || N < 0 || H < 0 || D < 0 || (!out && (int64_t)B * N * H * D > 0)) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 64) nthreads = 64;
  int64_t rows = (int64_t)B * N;
  fill_job jobs[64];
  pthread_t tids[64];
  for (int t = 0; t < nthreads; ++t) {
    fill_job* j = &jobs[t];
    j->key = stream_key(seed, stream);
    j->okey = stream_key(seed, outlier_stream);
    j->B = B; j->N = N; j->H = H; j->D = D;
    j->sb = sb; j->sn = sn; j->sh = sh;
    j->out = out; j->scale = scale; j->offset = hd_offset;
    j->oprob = outlier_prob; j->omult = outlier_mult;
    j->row_begin = rows * t / nthreads;
    j->row_end = rows * (t + 1) / nthreads;
  }
  int created[64] = {0};
  for (int t = 1; t < nthreads; ++t)
    created[t] = pthread_create(&tids[t], 0, fill_worker, &jobs[t]) == 0;
  fill_worker(&jobs[0]);
  for (int t = 1; t < nthreads; ++t) {
    if (created[t]) pthread_join(tids[t], 0);
    else fill_worker(&jobs[t]); /* could not start a thread: do its rows here */
  }
  return 0;
}

/* count uniform draws in [lo, hi) from one stream, as float. */
int synth_uniform_f32(uint64_t seed, uint32_t stream, int64_t count, float lo, float hi, float* out) {
  if (count < 0 || (!out && count > 0)) return -1;
  uint64_t key = stream_key(seed, stream);
  for (int64_t i = 0; i < count; ++i)
    out[i] = (float)((double)lo + ((double)hi - (double)lo) * uniform_at(key, (uint64_t)i));
  return 0;
}
