/*
 * Device fill routine of the synthetic input generator (definition in
 * synth_core.h).  Produces the same bits as synth_host.c: the multiply and
 * the planting add are written as separately rounded intrinsics so that the
 * compiler cannot contract them into one fused multiply-add.
 */
#include <cuda_runtime.h>
#include "synth_core.h"

namespace {

__global__ void fill_kernel(void* out, int dtype, long long a0, long long A, long long t0, long long t1, long long C,
                            long long stride_a, long long stride_t, unsigned long long key, float scale,
                            const float* delta, unsigned long long plant_key, unsigned plant_mod) {
  const long long T = t1 - t0;
  const long long cgroups = C / 8;  // C is a multiple of 8
  const long long total = A * T * cgroups;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    long long cg = e % cgroups;
    long long r = e / cgroups;
    long long t = t0 + r % T;
    long long a = a0 + r / T;
    bool plant = delta != nullptr && tbs_planted(plant_key, a, t, plant_mod);
    long long o = (a - a0) * stride_a + (t - t0) * stride_t + cg * 8;
    uint32_t packed[4];
    float vals[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      long long c = cg * 8 + j;
      float x = __fmul_rn(tbs_normal(key, tbs_index(a, t, c, C)), scale);
      if (plant) x = __fadd_rn(x, delta[a * C + c]);
      vals[j] = x;
    }
    if (dtype == 0) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        packed[j] = (uint32_t)tbs_bf16_rne(vals[2 * j]) | ((uint32_t)tbs_bf16_rne(vals[2 * j + 1]) << 16);
      *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + o) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    } else {
      float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o);
      p[0] = make_float4(vals[0], vals[1], vals[2], vals[3]);
      p[1] = make_float4(vals[4], vals[5], vals[6], vals[7]);
    }
  }
}

}  // namespace

/* Device version of tbs_fill_host (same arguments plus the stream).  `out`
 * points at element (a0, t0); `out` and `delta` are device pointers.  C must
 * be a multiple of 8 and every row start 16-byte aligned.
 * Returns 0, -1 on a bad argument, or the CUDA error code of the launch. */
extern "C" int tbs_fill_device(void* out, int dtype, long long a0, long long a1, long long t0, long long t1,
                               long long C,
                               long long stride_a, long long stride_t, unsigned long long key, float scale,
                               const float* delta, unsigned long long plant_key, unsigned plant_mod,
                               void* stream) {
  if (!out || a0 < 0 || a1 < a0 || t0 < 0 || t1 < t0 || C <= 0 || (C % 8) != 0 || (dtype != 0 && dtype != 1))
    return -1;
  long long A = a1 - a0;
  long long total = A * (t1 - t0) * (C / 8);
  if (total == 0) return 0;
  long long blocks = (total + 255) / 256;
  if (blocks > 148LL * 64) blocks = 148LL * 64;
  fill_kernel<<<(unsigned)blocks, 256, 0, (cudaStream_t)stream>>>(out, dtype, a0, A, t0, t1, C, stride_a, stride_t,
                                                                  key, scale, delta, plant_key, plant_mod);
  return (int)cudaGetLastError();
}
