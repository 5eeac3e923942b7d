// butler_attn_combine: the fp32 log-sum-exp merge of the sparse attention's
// split-K partials into each head's output row (and its log-sum-exp).
#pragma once

#include "attn.cuh"

namespace tb {

// ---------------------------------------------------------------- combine
struct CombineParams {
  const float* part_o;
  const float* part_ml;
  void* out;   // [B][Hq][D] kv dtype
  float* lse;  // [B][Hq] or nullptr
  int B, Hq, chunk, nsplit;
  int lens[kMaxBatch];
};

// fp32 log-sum-exp merge of the split partials: one CTA per (b, h).  All
// (m, l) pairs are loaded at once (one float2 each), together with each
// warp's first eight split rows; then each of the eight warps sums an eighth
// of the splits for the whole output row (lane = D/32 consecutive
// dimensions, eight split rows in flight per warp) and the eighths are added
// in shared memory.  An empty set gives out = 0 and lse = -inf.
constexpr int kCombineThreads = 256;
template <typename T, int D>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int DPL = D / 32;
  constexpr int NW = kCombineThreads / 32;
  __shared__ float sw[kMaxSplits];
  __shared__ float sred[NW][D];
  __shared__ float sM[NW], sS[NW];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int L = p.lens[b];
  const int ns = (L + p.chunk - 1) / p.chunk;
  const size_t ph = (size_t)bh * p.nsplit;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + ph;
  const float* po = p.part_o + ph * D + lane * DPL;
  // the warp's first kPre split rows are requested with the (m, l) pairs:
  // they do not depend on the merged maximum
  constexpr int kPre = 8;
  float pre[kPre][DPL];
#pragma unroll
  for (int i = 0; i < kPre; ++i) {
    const int sp = warp + i * NW;
#pragma unroll
    for (int e = 0; e < DPL; ++e) pre[i][e] = 0.f;
    if (sp < ns) {
      if constexpr (DPL == 4) {
        const float4 v = *reinterpret_cast<const float4*>(po + (size_t)sp * D);
        pre[i][0] = v.x;
        pre[i][1] = v.y;
        pre[i][2] = v.z;
        pre[i][3] = v.w;
      } else {
        const float2 v = *reinterpret_cast<const float2*>(po + (size_t)sp * D);
        pre[i][0] = v.x;
        pre[i][1] = v.y;
      }
    }
  }
  float M = kNegInf;
  float2 mine[(kMaxSplits + kCombineThreads - 1) / kCombineThreads];
#pragma unroll
  for (int r = 0; r < (kMaxSplits + kCombineThreads - 1) / kCombineThreads; ++r) {
    const int sp = tid + r * kCombineThreads;
    mine[r] = sp < ns ? ml[sp] : make_float2(kNegInf, 0.f);
    M = fmaxf(M, mine[r].x);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) sM[warp] = M;
  __syncthreads();
  M = sM[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, sM[w]);
  float lsum = 0.f;
#pragma unroll
  for (int r = 0; r < (kMaxSplits + kCombineThreads - 1) / kCombineThreads; ++r) {
    const int sp = tid + r * kCombineThreads;
    if (sp < ns) {
      const float f = (M == kNegInf || mine[r].x == kNegInf) ? 0.f : exp2f(mine[r].x - M);
      sw[sp] = f;
      lsum += f * mine[r].y;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if (lane == 0) sS[warp] = lsum;
  __syncthreads();
  lsum = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) lsum += sS[w];
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
#pragma unroll
  for (int i = 0; i < kPre; ++i) {
    const int sp = warp + i * NW;
    if (sp < ns) {
      const float w = sw[sp];
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[e] += w * pre[i][e];
    }
  }
#pragma unroll 8
  for (int sp = warp + kPre * NW; sp < ns; sp += NW) {
    const float w = sw[sp];
    if constexpr (DPL == 4) {
      const float4 v = *reinterpret_cast<const float4*>(po + (size_t)sp * D);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
      acc[2] += w * v.z;
      acc[3] += w * v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(po + (size_t)sp * D);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
    }
  }
#pragma unroll
  for (int i = 0; i < DPL; ++i) sred[warp][lane * DPL + i] = acc[i];
  __syncthreads();
  const float inv = M == kNegInf ? 0.f : 1.f / lsum;
  for (int d = tid; d < D; d += kCombineThreads) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) o += sred[w][d];
    reinterpret_cast<T*>(p.out)[(size_t)bh * D + d] = from_f32<T>(o * inv);
  }
  if (p.lse != nullptr && tid == 0) p.lse[bh] = M == kNegInf ? kNegInf : (M + log2f(lsum)) * 0.69314718055994531f;
}

}  // namespace tb
