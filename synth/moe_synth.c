/*
 * Seeded, counter-based generators for the synthetic inputs of the MoE layer.
 *
 * This file holds no arithmetic of the MoE method itself: it only draws the
 * random tensors (activations, router weights, expert weights and biases) that
 * both the CUDA path and the CPU oracle consume. Every value is a pure function
 * of (seed, stream, element index), so any slice of any tensor can be produced
 * on its own and the result does not depend on the number of threads.
 *
 *   key(seed, stream)   = mix64(mix64(seed + G) ^ (stream * S))
 *   draw(key, i)        = mix64(key + (i + 1) * G)          (splitmix64 finaliser)
 *   uniform(key, i)     = ((draw >> 11) + 0.5) * 2^-53        in (0, 1)
 *   normal(key, 2m+b)   = Box-Muller on (uniform(2m), uniform(2m+1)), cos for b=0, sin for b=1
 *
 * bf16 outputs are produced as double -> float (round to nearest even) ->
 * bf16 (round to nearest even on the top 16 bits).
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define SYNTH_G 0x9E3779B97F4A7C15ULL
#define SYNTH_S 0xD1B54A32D192ED03ULL

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return mix64(mix64(seed + SYNTH_G) ^ (stream * SYNTH_S));
}

static inline uint64_t draw(uint64_t key, uint64_t i) { return mix64(key + (i + 1) * SYNTH_G); }

static inline double uniform01(uint64_t key, uint64_t i) {
  return ((double)(draw(key, i) >> 11) + 0.5) * 0x1.0p-53;
}

static inline double normal01(uint64_t key, uint64_t i) {
  const uint64_t m = i >> 1;
  const double u1 = uniform01(key, 2 * m);
  const double u2 = uniform01(key, 2 * m + 1);
  const double r = sqrt(-2.0 * log(u1));
  const double a = 6.283185307179586476925286766559 * u2;
  return (i & 1) ? r * sin(a) : r * cos(a);
}

static inline uint16_t f32_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return (uint16_t)((u >> 16) | 0x40u);
  u += 0x7fffu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

/* Raw 64-bit draws (for tests of the generator itself). */
void synth_draw_u64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, uint64_t* out) {
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = draw(key, offset + (uint64_t)i);
}

void synth_uniform_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double* out) {
  const uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i) out[i] = uniform01(key, offset + (uint64_t)i);
}

/* Normal draws of elements [offset, offset + n): each Box-Muller pair (2m, 2m + 1) is formed once
 * and gives both of its elements (the same values as normal01 element by element). */
#define SYNTH_NORMAL_LOOP(STORE)                                                          \
  const uint64_t key = synth_key(seed, stream);                                           \
  if (n <= 0) return;                                                                     \
  const int64_t m0 = (int64_t)(offset >> 1), m1 = (int64_t)((offset + (uint64_t)n - 1) >> 1); \
  _Pragma("omp parallel for schedule(static)")                                            \
  for (int64_t m = m0; m <= m1; ++m) {                                                    \
    const double u1 = uniform01(key, 2 * (uint64_t)m);                                    \
    const double u2 = uniform01(key, 2 * (uint64_t)m + 1);                                \
    const double r = sqrt(-2.0 * log(u1));                                                \
    const double a = 6.283185307179586476925286766559 * u2;                               \
    for (int b = 0; b < 2; ++b) {                                                         \
      const uint64_t i = 2 * (uint64_t)m + (uint64_t)b;                                   \
      if (i < offset || i >= offset + (uint64_t)n) continue;                              \
      const double v = mean + std * (b ? r * sin(a) : r * cos(a));                        \
      STORE;                                                                              \
    }                                                                                     \
  }

void synth_normal_f64(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean,
                      double std, double* out) {
  SYNTH_NORMAL_LOOP(out[i - offset] = v)
}

void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean,
                      double std, float* out) {
  SYNTH_NORMAL_LOOP(out[i - offset] = (float)v)
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double mean,
                       double std, uint16_t* out) {
  SYNTH_NORMAL_LOOP(out[i - offset] = f32_to_bf16_bits((float)v))
}

/* A seeded permutation of 1..n (Fisher-Yates, swap index from draw % (i + 1)). */
void synth_permutation(uint64_t seed, uint64_t stream, int32_t n, int32_t* out) {
  const uint64_t key = synth_key(seed, stream);
  for (int32_t i = 0; i < n; ++i) out[i] = i + 1;
  for (int32_t i = n - 1; i > 0; --i) {
    const int32_t j = (int32_t)(draw(key, (uint64_t)i) % (uint64_t)(i + 1));
    const int32_t t = out[i];
    out[i] = out[j];
    out[j] = t;
  }
}
