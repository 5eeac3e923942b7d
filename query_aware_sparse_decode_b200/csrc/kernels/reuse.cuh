// Amortised selection: TokenButler's prediction interval and TokenSelect's
// selection cache (TokenButler abstract: importance predicted at intervals,
// with neighbouring tokens fetched; TokenSelect README, "Selection Cache":
// consecutive similar queries share selection results).  The pages give no
// numbers for the interval, the similarity test or the neighbourhood, so
// they are parameters: a row reuses its cached selection when
//   - the cache holds a selection made at length len0 > 0,
//   - len - len0 <= interval (tokens decoded since; the prediction interval),
//   - cos(q_hat_now, q_hat_cached) >= tau,
//   - and the row takes a real top-k (k strictly between 0 and the candidate
//     count) now.
// The reused set is the cached top-k (the cached mask restricted to
// [sink, len0 - window)), widened by `radius` neighbours on each side, kept
// inside the current candidates [sink, len - window), plus the current sink
// and window.  Other rows select afresh and refill the cache.
//
// reuse_decide_kernel: one warp per selection row (per query head, or per KV
// group with the group's importance queries summed in head order); fp32 dot
// products and norms by lane-ordered warp reductions.
#pragma once

#include "common.cuh"

namespace tb {

struct ReuseParams {
  const void* q_imp;   // [(B*Hq)][G][1][d'] of the producer, kv dtype
  float* sc_q;         // [B*rows][d']
  int32_t* sc_len;     // [B*rows]
  uint32_t* reuse;     // [B*rows] decisions of this step
  int G, slot, Hq, Hkv, rows_per_seq, nrows_total;
  float tau;
  int interval, keep_pct, sink, window;
  int lens[kMaxBatch];
};

template <typename T, int DIMP>
__global__ void __launch_bounds__(256) reuse_decide_kernel(const ReuseParams p) {
  pdl_wait();
  pdl_trigger();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 8 + warp;
  if (row >= p.nrows_total) return;  // warp-uniform
  const int b = row / p.rows_per_seq, r = row % p.rows_per_seq;
  const int L = p.lens[b];
  const int gs = p.rows_per_seq == p.Hq ? 1 : p.Hq / p.Hkv;  // heads summed into the row
  const T* qi = reinterpret_cast<const T*>(p.q_imp);
  float qv = 0.f, pv = 0.f;
  if (lane < DIMP) {
    const int h0 = gs == 1 ? r : r * gs;
    for (int hh = 0; hh < gs; ++hh)
      qv += to_f32(qi[(((size_t)b * p.Hq + h0 + hh) * p.G + p.slot) * DIMP + lane]);
    pv = p.sc_q[(size_t)row * DIMP + lane];
  }
  float dot = qv * pv, nq = qv * qv, np = pv * pv;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    dot += __shfl_xor_sync(0xffffffffu, dot, o);
    nq += __shfl_xor_sync(0xffffffffu, nq, o);
    np += __shfl_xor_sync(0xffffffffu, np, o);
  }
  const int len0 = p.sc_len[row];
  const int hi = L - p.window;
  const int nc = hi > p.sink ? hi - p.sink : 0;
  const long long k = min((long long)p.keep_pct * L / 100, (long long)nc);
  const bool topk_row = k > 0 && k < nc;
  const bool ok = topk_row && len0 > 0 && L >= len0 && L - len0 <= p.interval && nq > 0.f && np > 0.f &&
                  dot >= p.tau * sqrtf(nq * np);
  if (lane == 0) p.reuse[row] = ok ? 1u : 0u;
  if (!ok) {  // this step selects afresh: its query and length define the cache
    if (lane < DIMP) p.sc_q[(size_t)row * DIMP + lane] = qv;
    if (lane == 0) p.sc_len[row] = topk_row ? L : 0;  // only a real top-k is worth reusing
  }
}

// Bits i of the word starting at token `base` with a <= base + i < b.
__device__ __forceinline__ uint32_t range_bits(int base, int a, int b) {
  const int lo = max(a - base, 0), hi = min(b - base, 32);
  if (hi <= lo) return 0u;
  const uint32_t upto = hi >= 32 ? 0xFFFFFFFFu : ((1u << hi) - 1u);
  return upto & ~((1u << lo) - 1u);
}

}  // namespace tb
