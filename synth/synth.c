/*
 * Seeded, counter-based synthetic input generator.
 *
 * This module produces the input bytes that both the CUDA path and the fp64
 * CPU oracle consume.  It contains none of the attention arithmetic: it only
 * draws numbers.  Every element is a pure function of (seed, stream, index),
 * so any sub-range of a tensor can be generated on its own and in parallel.
 *
 * Definition (all arithmetic on unsigned 64-bit integers, wrapping):
 *   gamma    = 0x9E3779B97F4A7C15                 (SplitMix64 increment)
 *   mix(z)   = SplitMix64 output function (Steele, Lea & Flood, "Fast
 *              splittable pseudorandom number generators", OOPSLA 2014):
 *              z ^= z >> 30; z *= 0xBF58476D1CE4E5B9;
 *              z ^= z >> 27; z *= 0x94D049BB133111EB; z ^= z >> 31
 *   key      = mix(mix(seed) ^ ((stream + 1) * gamma))
 *   word(c)  = mix(key + (c + 1) * gamma)         (c = counter)
 *   unit(w)  = (w >> 11) * 2^-53                  in [0, 1)
 * Standard normal element i (Box-Muller, Box & Muller 1958):
 *   p = i >> 1, u1 = 1 - unit(word(2p)), u2 = unit(word(2p + 1)),
 *   R = sqrt(-2 ln u1), z = R cos(2 pi u2) for even i, R sin(2 pi u2) for odd i.
 * The value written is scale * z rounded to fp32 (C cast, round to nearest
 * even); bf16 outputs round that fp32 value to nearest even.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

static inline uint64_t synth_mix(uint64_t z) {
  z ^= z >> 30; z *= 0xBF58476D1CE4E5B9ULL;
  z ^= z >> 27; z *= 0x94D049BB133111EBULL;
  z ^= z >> 31;
  return z;
}

static inline uint64_t synth_key(uint64_t seed, uint64_t stream) {
  return synth_mix(synth_mix(seed) ^ ((stream + 1ULL) * SYNTH_GAMMA));
}

static inline uint64_t synth_word(uint64_t key, uint64_t c) {
  return synth_mix(key + (c + 1ULL) * SYNTH_GAMMA);
}

static inline double synth_unit(uint64_t w) {
  return (double)(w >> 11) * (1.0 / 9007199254740992.0);
}

static inline double synth_normal_at(uint64_t key, uint64_t i) {
  uint64_t p = i >> 1;
  double u1 = 1.0 - synth_unit(synth_word(key, 2 * p));
  double u2 = synth_unit(synth_word(key, 2 * p + 1));
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  return (i & 1ULL) ? r * sin(a) : r * cos(a);
}

/* fp32 -> bf16 bits, round to nearest even (NaN kept quiet). */
static inline uint16_t synth_f32_to_bf16(float f) {
  union { float f; uint32_t u; } v;
  v.f = f;
  if ((v.u & 0x7F800000u) == 0x7F800000u && (v.u & 0x007FFFFFu)) return (uint16_t)((v.u >> 16) | 0x40u);
  uint32_t lsb = (v.u >> 16) & 1u;
  v.u += 0x7FFFu + lsb;
  return (uint16_t)(v.u >> 16);
}

void synth_normal_f32(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double scale,
                      float* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) out[j] = (float)(scale * synth_normal_at(key, offset + (uint64_t)j));
}

void synth_normal_bf16(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double scale,
                       uint16_t* out) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j)
    out[j] = synth_f32_to_bf16((float)(scale * synth_normal_at(key, offset + (uint64_t)j)));
}

/* Integers uniform on [lo, hi]: lo + floor(unit(word(i)) * (hi - lo + 1)). */
void synth_uniform_int(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, int64_t lo,
                       int64_t hi, int64_t* out) {
  uint64_t key = synth_key(seed, stream);
  double span = (double)(hi - lo + 1);
  for (int64_t j = 0; j < n; ++j) {
    int64_t v = lo + (int64_t)floor(synth_unit(synth_word(key, offset + (uint64_t)j)) * span);
    out[j] = v > hi ? hi : v;
  }
}

/* Sparse ternary values in {-1, 0, +1}: element j is nonzero with probability
 * `density`, and then +1 or -1 with equal probability.  Written as bf16 bits
 * (or fp32 when out_f32 != NULL).  Used by the exact-integer tests. */
void synth_ternary(uint64_t seed, uint64_t stream, uint64_t offset, int64_t n, double density,
                   uint16_t* out_bf16, float* out_f32) {
  uint64_t key = synth_key(seed, stream);
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    uint64_t w = synth_word(key, offset + (uint64_t)j);
    double u = synth_unit(w);
    float v = 0.0f;
    if (u < density) v = (w & 1ULL) ? 1.0f : -1.0f;
    if (out_bf16) out_bf16[j] = synth_f32_to_bf16(v);
    if (out_f32) out_f32[j] = v;
  }
}

/* bf16 bits -> fp32 (exact widening). */
void synth_bf16_to_f32(const uint16_t* in, int64_t n, float* out) {
#pragma omp parallel for schedule(static)
  for (int64_t j = 0; j < n; ++j) {
    union { uint32_t u; float f; } v;
    v.u = ((uint32_t)in[j]) << 16;
    out[j] = v.f;
  }
}
