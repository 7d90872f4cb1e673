/*
 * Seeded synthetic-input generator: the one definition shared by the host
 * (synth_host.c) and device (synth_dev.cu) builds of this module.
 *
 * It produces the inputs of the ZeRO optimizer step -- per-rank bf16
 * gradient replicas and the initial fp32 master weights -- and nothing of
 * the step's own arithmetic (no reduction, no Adam, no rounding to bf16 by
 * nearest-even: a generated bf16 is the generated fp32 value truncated to its
 * upper 16 bits, which is this generator's own definition of its output).
 *
 * Counter-based draws: SplitMix64 (Steele, Lea & Flood, "Fast splittable
 * pseudorandom number generators", OOPSLA 2014).  The stream state for draw n
 * is `base + n * GAMMA` and the output is the SplitMix64 finaliser of that
 * state, so every element can be drawn independently on host or device.
 *
 * Element `idx` of stream `base` uses draws n = 5*idx + 1 .. 5*idx + 5:
 *   k = 0..3  four 24-bit uniforms for an Irwin-Hall(4) approximate normal,
 *             or k = 0 alone for a uniform value;
 *   k = 4     the exact-zero draw (value forced to 0 when draw % zero_mod == 0).
 */
#ifndef SYNTH_GEN_H
#define SYNTH_GEN_H

#include <stdint.h>

#if defined(__CUDACC__)
#define SYNTH_FN static __host__ __device__ __forceinline__
#else
#define SYNTH_FN static inline
#endif

#define SYNTH_GAMMA 0x9E3779B97F4A7C15ULL

enum { SYNTH_NORMAL = 0, SYNTH_UNIFORM = 1 };

SYNTH_FN uint64_t synth_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

/* Stream base for (seed, stream id, step, rank). */
SYNTH_FN uint64_t synth_base(uint64_t seed, uint32_t stream, uint32_t step,
                             uint32_t rank) {
  uint64_t h = synth_mix64(seed + SYNTH_GAMMA * (1ULL + (uint64_t)stream));
  h = synth_mix64(h ^ (0xD1B54A32D192ED03ULL * (1ULL + (uint64_t)step)));
  h = synth_mix64(h ^ (0x8CB92BA72F3D8DD7ULL * (1ULL + (uint64_t)rank)));
  return h;
}

SYNTH_FN uint64_t synth_draw(uint64_t base, int64_t idx, int k) {
  return synth_mix64(base + SYNTH_GAMMA * ((uint64_t)idx * 5ULL + (uint64_t)k + 1ULL));
}

/*
 * The fp32 value of element idx.
 *   SYNTH_NORMAL : c = sum_{k<4} (draw_k >> 40) - 2^25, value = (double)c * scale,
 *                  where the caller passes scale = sigma * sqrt(3) / 2^24
 *                  (unit variance before scaling; tails bounded at +-sqrt(12)/2*2 sigma).
 *   SYNTH_UNIFORM: value = ((draw_0 >> 40) * 2^-24 * 2 - 1) * scale, i.e. U(-scale, scale).
 * The double is rounded to fp32 by the ordinary conversion (round to nearest).
 */
SYNTH_FN float synth_value_f32(uint64_t base, int64_t idx, int kind, double scale,
                               uint32_t zero_mod) {
  if (zero_mod != 0u && (synth_draw(base, idx, 4) % (uint64_t)zero_mod) == 0ULL) return 0.0f;
  double x;
  if (kind == SYNTH_UNIFORM) {
    double u = (double)(synth_draw(base, idx, 0) >> 40) * (1.0 / 16777216.0);
    x = (u * 2.0 - 1.0) * scale;
  } else {
    int64_t c = 0;
    for (int k = 0; k < 4; ++k) c += (int64_t)(synth_draw(base, idx, k) >> 40);
    x = (double)(c - (int64_t)(1 << 25)) * scale;
  }
  return (float)x;
}

SYNTH_FN uint32_t synth_f32_bits(float f) {
  union { float f; uint32_t u; } c;
  c.f = f;
  return c.u;
}

/* Generated bf16 bit pattern: the fp32 value's upper half (truncation). */
SYNTH_FN uint16_t synth_value_bf16(uint64_t base, int64_t idx, int kind, double scale,
                                   uint32_t zero_mod) {
  return (uint16_t)(synth_f32_bits(synth_value_f32(base, idx, kind, scale, zero_mod)) >> 16);
}

/* Generated binary16 bit pattern: the fp32 value truncated toward zero to
 * IEEE binary16 (11-bit significand, subnormals spaced 2^-24, magnitudes from
 * 65504 up clamped to 65504) -- integer operations on the fp32 bits, this
 * generator's own definition of its fp16 output. */
SYNTH_FN uint16_t synth_f32_to_f16_trunc(float f) {
  const uint32_t u = synth_f32_bits(f);
  const uint16_t sign = (uint16_t)((u >> 16) & 0x8000u);
  const uint32_t a = u & 0x7FFFFFFFu;
  if (a >= 0x477FE000u) return (uint16_t)(sign | 0x7BFFu);
  const int e = (int)(a >> 23) - 127;
  if (e >= -14) return (uint16_t)(sign | (uint16_t)((e + 15) << 10) | (uint16_t)((a >> 13) & 0x3FFu));
  if (e < -25) return sign;
  const uint32_t mant = (a & 0x7FFFFFu) | 0x800000u;
  return (uint16_t)(sign | (uint16_t)(mant >> (uint32_t)(-(e + 1))));
}

SYNTH_FN uint16_t synth_value_f16(uint64_t base, int64_t idx, int kind, double scale, uint32_t zero_mod) {
  return synth_f32_to_f16_trunc(synth_value_f32(base, idx, kind, scale, zero_mod));
}

#endif /* SYNTH_GEN_H */
