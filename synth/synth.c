/*
 * Seeded synthetic inputs for the routed mixture-of-experts layer.
 *
 * This file builds INPUTS only: random activations, router weights, biases and
 * expert weights, plus the two storage encoders that turn a real-valued expert
 * matrix into the formats the layer consumes (int8 with one fp32 scale per
 * output row and expert; int4 in blocks of 32 with fp32 scales clamped at
 * 2^-14).  It holds none of the layer's arithmetic (no routing, no FFN, no
 * combine, no dequantisation), so both the fp64 oracle and the CUDA path can
 * consume what it writes without sharing any method code.
 *
 * Random numbers: a counter-based SplitMix64 stream.  Element i of stream s
 * under seed S is mix64(key(S, s) + (i + 1) * 0x9E3779B97F4A7C15), where mix64
 * is the SplitMix64 output function published by Steele, Lea and Flood
 * ("Fast splittable pseudorandom number generators", OOPSLA 2014).  Because
 * every element is a pure function of (S, s, i), a fill is identical for any
 * thread count.  Normals use the Box-Muller transform on consecutive pairs.
 *
 * Storage encoders (the pages' formats):
 *  - int8 per output channel: the routed experts carry one symmetric min-max
 *    scale per output row and expert -- Kimi-Linear LiteRT-LM details page,
 *    Conversion notes, quantization bullet.  s = max|w|/127,
 *    q = clamp(round_half_away(w/s), -127, 127); an all-zero row gets s = 1.
 *  - int4 block 32: blockwise int4 experts, 32 columns per fp32 scale, with
 *    scales under 2^-14 lifted to 2^-14 -- Qwen3-30B-A3B LiteRT-LM model card,
 *    Available Artifacts table and Conversion Notes.
 *    Blocks run along the reduction axis; s = max(max|w|/7, 2^-14),
 *    q = clamp(round_half_away(w/s), -8, 7), two's-complement nibbles, the
 *    low nibble holding the even column.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed + GOLDEN_GAMMA) ^ (stream * 0xD1B54A32D192ED03ULL));
}

static inline uint64_t draw_u64(uint64_t key, uint64_t i) {
  return mix64(key + (i + 1) * GOLDEN_GAMMA);
}

/* uniform in [0, 1) with 53 random bits */
static inline double draw_unit(uint64_t key, uint64_t i) {
  return (double)(draw_u64(key, i) >> 11) * (1.0 / 9007199254740992.0);
}

/* Box-Muller on the uniform pair (2j, 2j+1): z[0] is element 2j, z[1] element 2j+1 */
static inline void normal_pair(uint64_t key, uint64_t j, double z[2]) {
  const double u1 = 1.0 - draw_unit(key, 2 * j); /* (0, 1] */
  const double u2 = draw_unit(key, 2 * j + 1);
  const double r = sqrt(-2.0 * log(u1));
  const double a = 6.283185307179586476925286766559 * u2;
  z[0] = r * cos(a);
  z[1] = r * sin(a);
}

/* standard normal for element i */
static inline double draw_normal(uint64_t key, uint64_t i) {
  double z[2];
  normal_pair(key, i >> 1, z);
  return z[i & 1];
}

/* elements [lo, hi) of the normal stream, computing each pair once */
static void normal_range(uint64_t key, size_t lo, size_t hi, double* out) {
  size_t i = lo;
  if (i < hi && (i & 1)) out[0] = draw_normal(key, i++);
  for (; i + 1 < hi; i += 2) {
    double z[2];
    normal_pair(key, i >> 1, z);
    out[i - lo] = z[0];
    out[i - lo + 1] = z[1];
  }
  if (i < hi) out[i - lo] = draw_normal(key, i);
}

/* fp32 -> bf16 bits, round to nearest even (NaN kept quiet) */
static inline uint16_t f32_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  const uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------- */
/* thread fan-out over an index range                                          */

typedef struct job job;
typedef void (*job_fn)(const job*, size_t lo, size_t hi);
struct job {
  job_fn fn;
  void* out;
  void* out2;
  uint64_t key;
  double a, b;
  size_t rows, cols;
  size_t block; /* int4: quantisation block along the columns (32 or 128) */
};

typedef struct {
  const job* j;
  size_t lo, hi;
} slice;

static void* run_slice(void* p) {
  const slice* s = (const slice*)p;
  s->j->fn(s->j, s->lo, s->hi);
  return NULL;
}

static void fan_out(const job* j, size_t n, int nthreads) {
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if ((size_t)nthreads > n) nthreads = n ? (int)n : 1;
  if (nthreads == 1) {
    j->fn(j, 0, n);
    return;
  }
  pthread_t th[256];
  slice sl[256];
  for (int t = 0; t < nthreads; ++t) {
    sl[t].j = j;
    sl[t].lo = n * (size_t)t / (size_t)nthreads;
    sl[t].hi = n * (size_t)(t + 1) / (size_t)nthreads;
    if (pthread_create(&th[t], NULL, run_slice, &sl[t]) != 0) {
      run_slice(&sl[t]);
      th[t] = 0;
    }
  }
  for (int t = 0; t < nthreads; ++t)
    if (th[t]) pthread_join(th[t], NULL);
}

/* ------------------------------------------------------------------------- */
/* element fills                                                              */

#define CHUNK 4096

static void fill_normal_f32(const job* j, size_t lo, size_t hi) {
  float* o = (float*)j->out;
  double z[CHUNK];
  for (size_t c = lo; c < hi; c += CHUNK) {
    const size_t e = c + CHUNK < hi ? c + CHUNK : hi;
    normal_range(j->key, c, e, z);
    for (size_t i = c; i < e; ++i) o[i] = (float)(j->a + j->b * z[i - c]);
  }
}

static void fill_normal_bf16(const job* j, size_t lo, size_t hi) {
  uint16_t* o = (uint16_t*)j->out;
  double z[CHUNK];
  for (size_t c = lo; c < hi; c += CHUNK) {
    const size_t e = c + CHUNK < hi ? c + CHUNK : hi;
    normal_range(j->key, c, e, z);
    for (size_t i = c; i < e; ++i) o[i] = f32_to_bf16_bits((float)(j->a + j->b * z[i - c]));
  }
}

static void fill_uniform_f32(const job* j, size_t lo, size_t hi) {
  float* o = (float*)j->out;
  for (size_t i = lo; i < hi; ++i) o[i] = (float)(j->a + (j->b - j->a) * draw_unit(j->key, i));
}

static void fill_uniform_f64(const job* j, size_t lo, size_t hi) {
  double* o = (double*)j->out;
  for (size_t i = lo; i < hi; ++i) o[i] = j->a + (j->b - j->a) * draw_unit(j->key, i);
}

static inline double round_half_away(double v) { return v < 0 ? -floor(-v + 0.5) : floor(v + 0.5); }

/* rows [lo, hi) of a cols-wide N(0, std) matrix, each encoded int8 per row */
static void fill_int8_rows(const job* j, size_t lo, size_t hi) {
  int8_t* q = (int8_t*)j->out;
  float* s = (float*)j->out2;
  const size_t C = j->cols;
  float* w = (float*)malloc(C * sizeof(float));
  double* z = (double*)malloc(C * sizeof(double));
  for (size_t r = lo; r < hi; ++r) {
    double amax = 0.0;
    normal_range(j->key, r * C, r * C + C, z);
    for (size_t c = 0; c < C; ++c) {
      w[c] = (float)(j->b * z[c]);
      const double a = fabs((double)w[c]);
      if (a > amax) amax = a;
    }
    const float sc = amax > 0.0 ? (float)(amax / 127.0) : 1.0f;
    s[r] = sc;
    for (size_t c = 0; c < C; ++c) {
      double v = round_half_away((double)w[c] / (double)sc);
      if (v > 127.0) v = 127.0;
      if (v < -127.0) v = -127.0;
      q[r * C + c] = (int8_t)v;
    }
  }
  free(w);
  free(z);
}

/* rows [lo, hi) of a cols-wide N(0, std) matrix, int4 blocks of 32 along cols */
static void fill_int4_blocks(const job* j, size_t lo, size_t hi) {
  uint8_t* q = (uint8_t*)j->out;
  float* s = (float*)j->out2;
  const size_t B = j->block, C = j->cols, NB = C / B;
  const double floor_scale = 1.0 / 16384.0; /* 2^-14 */
  float w[128];
  double z[128];
  for (size_t r = lo; r < hi; ++r) {
    for (size_t bi = 0; bi < NB; ++bi) {
      double amax = 0.0;
      normal_range(j->key, r * C + bi * B, r * C + bi * B + B, z);
      for (size_t c = 0; c < B; ++c) {
        w[c] = (float)(j->b * z[c]);
        const double a = fabs((double)w[c]);
        if (a > amax) amax = a;
      }
      double scd = amax / 7.0;
      if (scd < floor_scale) scd = floor_scale;
      float sc = (float)scd;
      if ((double)sc < floor_scale) sc = (float)floor_scale;
      s[r * NB + bi] = sc;
      for (size_t c = 0; c < B; c += 2) {
        int v[2];
        for (int h = 0; h < 2; ++h) {
          double t = round_half_away((double)w[c + h] / (double)sc);
          if (t > 7.0) t = 7.0;
          if (t < -8.0) t = -8.0;
          v[h] = (int)t;
        }
        q[r * (C / 2) + (bi * B + c) / 2] = (uint8_t)((v[0] & 0xF) | ((v[1] & 0xF) << 4));
      }
    }
  }
}

/* ------------------------------------------------------------------------- */
/* exported entry points (all return 0 on success, -1 on bad arguments)        */

int synth_normal_f32(float* out, size_t n, uint64_t seed, uint64_t stream, double mean, double std,
                     int nthreads) {
  if (!out && n) return -1;
  job j = {fill_normal_f32, out, NULL, stream_key(seed, stream), mean, std, 0, 0};
  fan_out(&j, n, nthreads);
  return 0;
}

int synth_normal_bf16(uint16_t* out, size_t n, uint64_t seed, uint64_t stream, double mean,
                      double std, int nthreads) {
  if (!out && n) return -1;
  job j = {fill_normal_bf16, out, NULL, stream_key(seed, stream), mean, std, 0, 0};
  fan_out(&j, n, nthreads);
  return 0;
}

int synth_uniform_f32(float* out, size_t n, uint64_t seed, uint64_t stream, double lo, double hi,
                      int nthreads) {
  if (!out && n) return -1;
  job j = {fill_uniform_f32, out, NULL, stream_key(seed, stream), lo, hi, 0, 0};
  fan_out(&j, n, nthreads);
  return 0;
}

int synth_uniform_f64(double* out, size_t n, uint64_t seed, uint64_t stream, double lo, double hi) {
  if (!out && n) return -1;
  job j = {fill_uniform_f64, out, NULL, stream_key(seed, stream), lo, hi, 0, 0};
  fan_out(&j, n, 1);
  return 0;
}

/* q: [rows, cols] int8, s: [rows] fp32 */
int synth_int8_rows(int8_t* q, float* s, size_t rows, size_t cols, uint64_t seed, uint64_t stream,
                    double std, int nthreads) {
  if ((!q || !s) && rows) return -1;
  job j = {fill_int8_rows, q, s, stream_key(seed, stream), 0.0, std, rows, cols};
  fan_out(&j, rows, nthreads);
  return 0;
}

/* q: [rows, cols/2] packed nibbles, s: [rows, cols/block] fp32; block 32 or 128,
   cols % block == 0.  The real-valued weights do not depend on the block size. */
int synth_int4_blocks_b(uint8_t* q, float* s, size_t rows, size_t cols, size_t block, uint64_t seed,
                        uint64_t stream, double std, int nthreads) {
  if (((!q || !s) && rows) || (block != 32 && block != 128) || cols % block) return -1;
  job j = {fill_int4_blocks, q, s, stream_key(seed, stream), 0.0, std, rows, cols, block};
  fan_out(&j, rows, nthreads);
  return 0;
}

int synth_int4_blocks(uint8_t* q, float* s, size_t rows, size_t cols, uint64_t seed, uint64_t stream,
                      double std, int nthreads) {
  return synth_int4_blocks_b(q, s, rows, cols, 32, seed, stream, std, nthreads);
}

/* raw stream access, for checking the generator itself */
uint64_t synth_draw_u64(uint64_t seed, uint64_t stream, uint64_t i) {
  return draw_u64(stream_key(seed, stream), i);
}
