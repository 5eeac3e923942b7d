/*
 * Host fill routine of the synthetic input generator (definition in
 * synth_core.h).  Build with -ffp-contract=off so that the multiply by
 * `scale` and the planting add stay two separately rounded IEEE operations,
 * as on the device.
 */
#include "synth_core.h"

/* out[(a - a0) * stride_a + (t - t0) * stride_t + c] for a0 <= a < a1,
 * t0 <= t < t1, c < C.  dtype 0: bf16 bits (uint16), 1: fp32.
 * delta: fp32 indexed delta[a * C + c] (absolute a) or NULL.
 * Returns 0, or -1 on a bad argument. */
int tbs_fill_host(void* out, int dtype, int64_t a0, int64_t a1, int64_t t0, int64_t t1, int64_t C,
                  int64_t stride_a, int64_t stride_t, uint64_t key, float scale,
                  const float* delta, uint64_t plant_key, uint32_t plant_mod) {
  if (!out || a0 < 0 || a1 < a0 || t0 < 0 || t1 < t0 || C <= 0 || (dtype != 0 && dtype != 1)) return -1;
#pragma omp parallel for collapse(2) schedule(static)
  for (int64_t a = a0; a < a1; ++a) {
    for (int64_t t = t0; t < t1; ++t) {
      int plant = delta != 0 && tbs_planted(plant_key, (uint64_t)a, (uint64_t)t, plant_mod);
      for (int64_t c = 0; c < C; ++c) {
        float x = tbs_normal(key, tbs_index((uint64_t)a, (uint64_t)t, (uint64_t)c, (uint64_t)C)) * scale;
        if (plant) x = x + delta[a * C + c];
        int64_t o = (a - a0) * stride_a + (t - t0) * stride_t + c;
        if (dtype == 0) ((uint16_t*)out)[o] = tbs_bf16_rne(x);
        else ((float*)out)[o] = x;
      }
    }
  }
  return 0;
}

/* flags[a * (t1 - t0) + (t - t0)] = planted(a, t) */
int tbs_planted_host(uint8_t* flags, int64_t A, int64_t t0, int64_t t1, uint64_t plant_key,
                     uint32_t plant_mod) {
  if (!flags || A < 0 || t1 < t0) return -1;
  for (int64_t a = 0; a < A; ++a)
    for (int64_t t = t0; t < t1; ++t)
      flags[a * (t1 - t0) + (t - t0)] = (uint8_t)tbs_planted(plant_key, (uint64_t)a, (uint64_t)t, plant_mod);
  return 0;
}

uint64_t tbs_stream_key_host(uint64_t seed, uint64_t stream) { return tbs_stream_key(seed, stream); }
