// Prefill row selection: for every query position p of a prefill chunk and
// every query head, score the causal prefix with that position's importance
// query and keep top-k + sink + window with L -> p + 1 (model card
// "Meta-Llama-3.1-8B-Instruct-Butler", section "Method": each consumer scores
// the cached tokens with its producer's importance query, slot (l - 1) mod G,
// and keeps a top-x subset under a fixed budget plus the sink prefix and the
// local window).
//
// One 1024-thread CTA per (b, h, row): the row's fp32 scores (t <= p) are
// computed once from K_imp (fp32 FMA) into shared memory, the k-th largest
// order key is found by the same three-digit radix select as the decode
// selection, and an ordered sweep writes the row's bitmask.
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace tb {

struct PrefillParams {
  const void* q_imp;   // [(B*Hq)][G][nrows][d'] kv dtype
  const float* kimp;   // [B][Hkv][max_len/256][d'][256] (kimp_index)
  uint32_t* masks;     // [B][Hq][nrows][words_per_row]
  uint32_t* status;
  int G, slot, Hq, Hkv, max_len, row0, nrows, words_per_row;
  int keep_pct, sink, window;
};

template <typename TQ, int DIMP>
__global__ void __launch_bounds__(kSelThreads, 1) prefill_select_kernel(const PrefillParams p) {
  extern __shared__ float srow[];  // scores of t <= row position
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  __shared__ float q[DIMP];
  const int r = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31;
  const int gs = p.Hq / p.Hkv, g = h / gs;
  const int pos = p.row0 + r;
  const int L = pos + 1;
  if (tid < DIMP)
    q[tid] = to_f32(reinterpret_cast<const TQ*>(p.q_imp)[((((size_t)b * p.Hq + h) * p.G + p.slot) * p.nrows + r) * DIMP +
                                                         tid]);
  __syncthreads();
  const size_t slab = (size_t)b * p.Hkv + g;
  for (int t = tid; t < L; t += kSelThreads) {
    const float* K = p.kimp + kimp_index(slab, 0, t, DIMP, p.max_len);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < DIMP; ++j) acc = fmaf(q[j], K[j * kKimpTile], acc);
    srow[t] = acc;
  }
  __syncthreads();

  const int lo = p.sink, hi = L - p.window;
  const int nc = hi > lo ? hi - lo : 0;
  const int k = (int)min((long long)p.keep_pct * L / 100, (long long)nc);
  uint32_t T = 0, quota = 0;
  int mode = 0;
  if (k == nc && k > 0) mode = 1;
  if (k > 0 && k < nc) {
    mode = 2;
    uint32_t prefix = 0, kk = (uint32_t)k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbits = pass == 2 ? 10 : 11;
      const int pshift = pass == 1 ? 21 : 10;
      for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int base = lo; base < hi; base += kSelThreads) {
        const int t = base + tid;
        const bool inr = t < hi;
        const uint32_t key = order_key(inr ? srow[t] : 0.f);
        const bool in = inr && (pass == 0 || (key >> pshift) == prefix);
        const uint32_t bin = in ? ((key >> shift) & ((1u << nbits) - 1)) : 0xFFFFFFFFu;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
      __syncthreads();
      if (pass < 2)
        find_bin<2>(hist, kk, scan_sm, &s_bin, &s_above);
      else
        find_bin<1>(hist, kk, scan_sm, &s_bin, &s_above);
      kk -= s_above;
      prefix = (prefix << nbits) | (uint32_t)s_bin;
      __syncthreads();
    }
    T = prefix;
    quota = kk;
  }

  // ordered sweep: 32 tokens per warp step, one bit per lane, ballot = mask word
  uint32_t* mrow = p.masks + ((((size_t)b * p.Hq + h) * p.nrows + r) * p.words_per_row);
  uint32_t tie_base = 0, count = 0;
  for (int base = 0; base < p.words_per_row * 32; base += kSelThreads) {
    const int t = base + tid;
    bool keep = false, tie = false;
    if (t < L) {
      const bool cand = t >= lo && t < hi;
      keep = !cand;
      if (cand && mode == 1) keep = true;
      if (cand && mode == 2) {
        const uint32_t key = order_key(srow[t]);
        if (key > T) keep = true;
        else if (key == T) tie = true;
      }
    }
    uint32_t total;
    const uint32_t ex = block_excl_scan<kSelThreads>(tie ? 1u : 0u, total, scan_sm);
    if (tie && tie_base + ex < quota) keep = true;
    tie_base += total;
    const uint32_t word = __ballot_sync(0xffffffffu, keep);
    if (lane == 0 && (t >> 5) < p.words_per_row) mrow[t >> 5] = word;
    count += __popc(word) * (lane == 0);
  }
  // count check: every warp's lane 0 holds a partial count
  uint32_t tot;
  (void)block_excl_scan<kSelThreads>(count, tot, scan_sm);
  if (tid == 0) {
    const int sink_n = min(p.sink, L);
    const int win_lo = max(L - p.window, sink_n);
    if (tot != (uint32_t)(sink_n + (L - win_lo) + k)) atomicOr(p.status, TB_DEV_ERR_COUNT);
  }
}

}  // namespace tb
