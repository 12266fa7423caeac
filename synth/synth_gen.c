/*
 * Seeded, counter-based synthetic input generator.
 *
 * This file holds no arithmetic of the mixture-of-experts layer: it only
 * turns (seed, tensor id, element index) into a normally distributed number
 * and rounds it to the storage type.  Both the GPU path's tests/benchmark and
 * the CPU oracle consume the bytes it writes, so the two sides see identical
 * inputs.
 *
 * Definition (fixed; any change alters every input):
 *   mix(z)      = splitmix64 finaliser:
 *                 z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *                 z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
 *   base(s, id) = mix(mix(s + G) ^ (id * 0xD1B54A32D192ED03))   G = 0x9E3779B97F4A7C15
 *   word(n)     = mix(base + (n + 1) * G)
 *   u1          = ((word(2i) >> 11) + 1) * 2^-53        in (0, 1]
 *   u2          =  (word(2i+1) >> 11)    * 2^-53        in [0, 1)
 *   z_i         = sqrt(-2 ln u1) * cos(2 pi u2)         (Box-Muller, cosine branch)
 *   value_i     = mean + sigma * z_i, computed in double, then rounded
 *                 to bfloat16 (round to nearest, ties to even) or float.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ULL

static inline uint64_t mix64(uint64_t z) {
  z ^= z >> 30;
  z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27;
  z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t stream_base(uint64_t seed, uint64_t tensor_id) {
  return mix64(mix64(seed + GOLDEN) ^ (tensor_id * 0xD1B54A32D192ED03ULL));
}

static inline double normal_at(uint64_t base, uint64_t i) {
  const double two_m53 = 1.1102230246251565404e-16; /* 2^-53 */
  uint64_t w1 = mix64(base + (2 * i + 1) * GOLDEN);
  uint64_t w2 = mix64(base + (2 * i + 2) * GOLDEN);
  double u1 = (double)((w1 >> 11) + 1) * two_m53;
  double u2 = (double)(w2 >> 11) * two_m53;
  return sqrt(-2.0 * log(u1)) * cos(6.283185307179586476925 * u2);
}

/* float -> bfloat16 bits, round to nearest even (NaN is never produced here). */
static inline uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

/* double -> bfloat16 with a single rounding: round the double to the bf16
 * grid directly (via float is double rounding; avoid it by rounding on the
 * double's bits). */
static inline uint16_t f64_to_bf16_rne(double v) {
  /* A bf16 has 8 significant bits.  Round the double to 8 significant bits
   * (RNE), which is then exactly representable as float and as bf16. */
  if (v == 0.0) return (uint16_t)(signbit(v) ? 0x8000u : 0u);
  int e;
  double m = frexp(v, &e);           /* v = m * 2^e, 0.5 <= |m| < 1 */
  double scaled = ldexp(m, 8);       /* 8 significant bits in the integer part */
  double r = nearbyint(scaled);      /* default rounding mode: ties to even */
  float f = (float)ldexp(r, e - 8);  /* exact */
  return f32_to_bf16_rne(f);         /* exact, no further rounding */
}

/* Fill out[i] (bf16 bits) for i in [0, n). */
void synth_normal_bf16(uint64_t seed, uint64_t tensor_id, int64_t n, double mean,
                       double sigma, uint16_t *out) {
  uint64_t base = stream_base(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = f64_to_bf16_rne(mean + sigma * normal_at(base, (uint64_t)i));
}

/* Fill out[i] (float) for i in [0, n). */
void synth_normal_f32(uint64_t seed, uint64_t tensor_id, int64_t n, double mean,
                      double sigma, float *out) {
  uint64_t base = stream_base(seed, tensor_id);
#pragma omp parallel for schedule(static)
  for (int64_t i = 0; i < n; ++i)
    out[i] = (float)(mean + sigma * normal_at(base, (uint64_t)i));
}

/* Raw 64-bit words, exposed so tests can pin the generator to its definition. */
void synth_words(uint64_t seed, uint64_t tensor_id, int64_t n, uint64_t *out) {
  uint64_t base = stream_base(seed, tensor_id);
  for (int64_t i = 0; i < n; ++i) out[i] = mix64(base + ((uint64_t)i + 1) * GOLDEN);
}
