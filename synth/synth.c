/*
 * Seeded synthetic-input generator shared by the tests, the benchmark and the
 * oracle checks.  It holds none of the attention method's arithmetic: it only
 * draws Gaussian numbers and rounds them to bfloat16 or float32.
 *
 * Generator: counter-based SplitMix64 (G. L. Steele, D. Lea, C. H. Flood,
 * "Fast splittable pseudorandom number generators", OOPSLA 2014).  Draw i of
 * stream s under seed k is mix(key(k, s) + (i + 1) * GAMMA), so any sub-range of
 * a stream can be produced independently and in parallel.  The 64 output bits
 * are split into two 32-bit uniforms (u1, u2) in (0, 1) and turned into one
 * standard normal by the Box-Muller transform z = sqrt(-2 ln u1) cos(2 pi u2)
 * (G. E. P. Box, M. E. Muller, Ann. Math. Statist. 29, 1958), in double.
 *
 * Rounding: double -> float (round to nearest even) -> bfloat16 (round to
 * nearest even on the top 16 bits).  Values are finite, so no NaN handling.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

static inline uint64_t stream_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed + GAMMA) + (stream + 1) * 0xD1B54A32D192ED03ULL);
}

static inline double normal_at(uint64_t key, uint64_t i) {
  uint64_t b = mix64(key + (i + 1) * GAMMA);
  double u1 = ((double)(uint32_t)(b >> 32) + 0.5) * (1.0 / 4294967296.0);
  double u2 = ((double)(uint32_t)(b & 0xFFFFFFFFu) + 0.5) * (1.0 / 4294967296.0);
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* out[i] = bf16( sigma * z(start + i) + (offset ? offset[i % period] : 0) ),  i in [0, n). */
void synth_normal_bf16(uint16_t* out, int64_t n, uint64_t seed, uint64_t stream, int64_t start,
                       double sigma, const float* offset, int64_t period) {
  const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) {
    double v = sigma * normal_at(key, (uint64_t)(start + i));
    if (offset) v += (double)offset[i % period];
    out[i] = f32_to_bf16_rne((float)v);
  }
}

/* out[i] = float( sigma * z(start + i) ),  i in [0, n). */
void synth_normal_f32(float* out, int64_t n, uint64_t seed, uint64_t stream, int64_t start,
                      double sigma) {
  const uint64_t key = stream_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = (float)(sigma * normal_at(key, (uint64_t)(start + i)));
}

/* A uniform integer in [0, m) from draw `i` of a stream (used to pick pages/segments). */
int64_t synth_uniform_int(uint64_t seed, uint64_t stream, int64_t i, int64_t m) {
  uint64_t b = mix64(stream_key(seed, stream) + ((uint64_t)i + 1) * GAMMA);
  return (int64_t)(b % (uint64_t)m);
}
