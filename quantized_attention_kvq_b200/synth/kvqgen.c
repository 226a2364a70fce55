/*
 * Seeded synthetic inputs for the quantized-KV decode path.
 *
 * This module only draws random numbers and rounds them to the storage
 * format a caller asks for (fp32 or bf16).  It holds none of the method's
 * arithmetic (no rotation, no quantization, no attention), so both the CUDA
 * path and the CPU oracle can consume the very same host arrays.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014).  The n-th output of a SplitMix64 stream
 * seeded with `key` is mix(key + n * 0x9E3779B97F4A7C15), so every element can
 * be drawn from its own counter and any slice of a tensor can be regenerated
 * on its own.  Normals come from the cosine branch of the Box-Muller transform
 * in fp64, one normal per pair of counters.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* n-th output (n >= 1) of the SplitMix64 stream seeded with key */
uint64_t kvqgen_u64(uint64_t key, uint64_t n) { return mix64(key + n * GOLDEN); }

/* stream key for one named tensor of one workload */
uint64_t kvqgen_key(uint64_t seed, uint64_t tag) { return kvqgen_u64(seed, tag + 1); }

static inline double unit_open0(uint64_t x) { return (double)((x >> 11) + 1) * 0x1.0p-53; } /* (0,1] */
static inline double unit_closed0(uint64_t x) { return (double)(x >> 11) * 0x1.0p-53; }     /* [0,1) */

/* i-th standard normal of stream `key` (i >= 0) */
double kvqgen_normal(uint64_t key, uint64_t i) {
  const double two_pi = 6.283185307179586476925286766559;
  double u1 = unit_open0(kvqgen_u64(key, 2 * i + 1));
  double u2 = unit_closed0(kvqgen_u64(key, 2 * i + 2));
  return sqrt(-2.0 * log(u1)) * cos(two_pi * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/*
 * out[e] = fmt(normal(key, first + e) * (scale ? scale[e % period] : 1)),
 * e in [0, count).  The product is formed in fp64, rounded to fp32 and, for
 * fmt == 1, rounded again (nearest-even) to bf16.  fmt 0 = fp32, 1 = bf16.
 */
void kvqgen_fill(uint64_t key, uint64_t first, int64_t count, const double* scale, int64_t period,
                 int32_t fmt, void* out) {
#pragma omp parallel for schedule(static)
  for (int64_t e = 0; e < count; ++e) {
    double v = kvqgen_normal(key, first + (uint64_t)e);
    if (scale) v *= scale[e % period];
    float f = (float)v;
    if (fmt == 1)
      ((uint16_t*)out)[e] = f32_to_bf16_rne(f);
    else
      ((float*)out)[e] = f;
  }
}

/*
 * Per-channel key scales of one KV head: c[ch] = exp(sigma * N(0,1)); then
 * n_outliers distinct channels (partial Fisher-Yates shuffle driven by the
 * same stream) are multiplied by outlier_mult.
 */
void kvqgen_chscale(uint64_t key, int32_t d, double sigma, int32_t n_outliers, double outlier_mult,
                    double* out) {
  int32_t idx[4096];
  if (d > 4096) return;
  for (int32_t c = 0; c < d; ++c) {
    out[c] = exp(sigma * kvqgen_normal(key, (uint64_t)c));
    idx[c] = c;
  }
  for (int32_t i = 0; i < n_outliers && i < d; ++i) {
    uint64_t r = kvqgen_u64(key, 0x100000000ULL + (uint64_t)i);
    int32_t j = i + (int32_t)(r % (uint64_t)(d - i));
    int32_t t = idx[i];
    idx[i] = idx[j];
    idx[j] = t;
    out[idx[i]] *= outlier_mult;
  }
}

/* out[b] uniform integer in [lo, hi] */
void kvqgen_lengths(uint64_t key, int32_t count, int32_t lo, int32_t hi, int32_t* out) {
  uint64_t span = (uint64_t)(hi - lo) + 1;
  for (int32_t b = 0; b < count; ++b) out[b] = lo + (int32_t)(kvqgen_u64(key, (uint64_t)b + 1) % span);
}
