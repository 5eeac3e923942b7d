/*
 * Counter-based synthetic input generator, shared by the host (C) and the
 * device (CUDA) fill routines so that both produce the same bits.
 *
 * This file holds no step of the decode method: it only turns
 * (seed, stream, coordinates) into input values.
 *
 * Definition
 *   mix64(z)          SplitMix64 finaliser (Steele, Lea, Flood, "Fast
 *                     splittable pseudorandom number generators", 2014;
 *                     constants of Vigna's splitmix64.c).
 *   key(seed, s)      = mix64(seed * PHI + s)                    (mod 2^64)
 *   i(a, t, c; C)     = ((a << 32) + t) * C + c                   logical index
 *   w_j               = mix64(key + (3 i + j + 1) * PHI),  j = 0, 1, 2
 *   S                 = sum of the twelve 16-bit fields of w_0, w_1, w_2
 *   z                 = (S + 6 - 6 * 65536) / 65536               (exact in fp32)
 * z is an Irwin-Hall(12) draw: mean 0, variance 1, support (-6, 6).
 * x = z * scale is one IEEE fp32 multiply (round to nearest even); a planted
 * element adds one fp32 value delta with one IEEE fp32 add.  bf16 outputs are
 * rounded from fp32 to nearest even by integer arithmetic on the bits.
 */
#ifndef TB_SYNTH_CORE_H
#define TB_SYNTH_CORE_H

#include <stdint.h>
#include <string.h>

#ifdef __CUDACC__
#define TBS_FN __host__ __device__ __forceinline__
#else
#define TBS_FN static inline
#endif

#define TBS_PHI 0x9E3779B97F4A7C15ULL

TBS_FN uint64_t tbs_mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
  return z ^ (z >> 31);
}

TBS_FN uint64_t tbs_stream_key(uint64_t seed, uint64_t stream) {
  return tbs_mix64(seed * TBS_PHI + stream);
}

TBS_FN uint64_t tbs_index(uint64_t a, uint64_t t, uint64_t c, uint64_t C) {
  return ((a << 32) + t) * C + c;
}

/* Irwin-Hall(12) value n / 65536 with |n| < 2^19: the int->float conversion
 * and the power-of-two scaling are both exact. */
TBS_FN float tbs_normal(uint64_t key, uint64_t i) {
  int32_t s = 0;
  for (int j = 0; j < 3; ++j) {
    uint64_t w = tbs_mix64(key + (3ULL * i + (uint64_t)j + 1ULL) * TBS_PHI);
    s += (int32_t)(w & 0xFFFFu) + (int32_t)((w >> 16) & 0xFFFFu) +
         (int32_t)((w >> 32) & 0xFFFFu) + (int32_t)(w >> 48);
  }
  return (float)(s + 6 - 393216) * (1.0f / 65536.0f);
}

/* planted(a, t) iff mix64(plant_key + ((a << 32) + t) * PHI) mod m == 0 */
TBS_FN int tbs_planted(uint64_t plant_key, uint64_t a, uint64_t t, uint32_t m) {
  if (m == 0) return 0;
  return (tbs_mix64(plant_key + ((a << 32) + t) * TBS_PHI) % (uint64_t)m) == 0;
}

TBS_FN uint32_t tbs_f32_bits(float f) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(f);
#else
  uint32_t u;
  memcpy(&u, &f, 4);
  return u;
#endif
}

/* fp32 -> bf16 bits, round to nearest even (finite inputs only) */
TBS_FN uint16_t tbs_bf16_rne(float f) {
  uint32_t u = tbs_f32_bits(f);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

#endif /* TB_SYNTH_CORE_H */
