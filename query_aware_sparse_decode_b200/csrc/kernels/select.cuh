// butler_topk + butler_merge: per (b, row) selection under a fixed budget
// (model card "Meta-Llama-3.1-8B-Instruct-Butler", section "Method": top-x
// subset under a fixed token budget plus a sink prefix and a recent local
// window; section "Memory requirements": fixed_<N>pc, min_sparse_index,
// sliding_window).
//
//   k = floor(P * L / 100), candidates C = [sink, L - window),
//   Sel = [0, min(sink, L)) U top_min(k, |C|)(C) U [max(L - window, 0), L),
//   order (score desc, index asc), -0.0 == +0.0.
//
// One 1024-thread CTA per row.  The k-th largest order key T is found by a
// three-digit radix select (11 + 11 + 10 bits): shared-memory histograms
// filled with warp-aggregated atomics (__match_any_sync + popc), each digit
// chosen by a block-wide suffix scan.  The first digit's histogram can come
// from the score kernel.  A final ordered sweep keeps keys > T and the
// lowest-index `quota` keys == T, writing the ascending index list and the
// bitmask with ballot/shuffle packing; the sink and window are merged in the
// same sweep, so the output is ascending by construction.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kSelThreads = 1024;

struct SelectParams {
  const float* scores;     // row r of sequence b at (b * rows_per_seq + r) * row_stride
  const uint32_t* hist1;   // [B*rows][2048] first-digit histograms, or nullptr
  int32_t* idx;            // [B*rows][idx_cap] or nullptr
  int32_t* count;          // [B*rows] or nullptr
  uint32_t* mask;          // [B*rows][mask_words] or nullptr
  uint32_t* status;
  long long row_stride;
  int rows_per_seq, idx_cap, mask_words;
  int keep_pct, sink, window;
  int lens[kMaxBatch];
};

// Find the bin b (scanning from the top) where the running count reaches k:
// sum(bins > b) < k <= sum(bins >= b).  NB bins, PER = NB / 1024 per thread.
template <int PER>
__device__ __forceinline__ void find_bin(const uint32_t* hist, uint32_t k, uint32_t* scan_sm, int* out_bin,
                                         uint32_t* out_above) {
  constexpr int NB = PER * kSelThreads;
  const int tid = threadIdx.x;
  uint32_t c[PER];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    c[j] = hist[NB - 1 - (tid * PER + j)];  // descending bin order
    local += c[j];
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan<kSelThreads>(local, total, scan_sm);
  if (excl < k && k <= excl + local) {
    uint32_t run = excl;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (run + c[j] >= k) {
        *out_bin = NB - 1 - (tid * PER + j);
        *out_above = run;
        break;
      }
      run += c[j];
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelectParams p) {
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const int r = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int L = p.lens[b];
  const long long row = (long long)b * p.rows_per_seq + r;
  const float* s = p.scores + row * p.row_stride;
  const int lo = p.sink, hi = L - p.window;
  const int nc = hi > lo ? hi - lo : 0;
  const int k = (int)min((long long)p.keep_pct * L / 100, (long long)nc);

  // ---- radix select of the k-th largest key among the candidates
  uint32_t T = 0, quota = 0;
  int mode = 0;  // 0: no candidate kept, 1: all kept, 2: threshold T + quota ties
  if (k == nc && k > 0) mode = 1;
  if (k > 0 && k < nc) {
    mode = 2;
    uint32_t prefix = 0, kk = (uint32_t)k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
      const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
      const int nbits = pass == 2 ? 10 : 11;
      const int pshift = pass == 1 ? 21 : 10;  // compare key >> pshift with prefix (passes 1, 2)
      if (pass == 0 && p.hist1 != nullptr) {
        for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = p.hist1[row * kHistBins + i];
        __syncthreads();
      } else {
        for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int base = lo & ~3; base < hi; base += 4 * kSelThreads) {
          const int t0 = base + 4 * tid;
          float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
          if (t0 < hi) v = *reinterpret_cast<const float4*>(s + t0);
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int t = t0 + j;
            const uint32_t key = order_key(vv[j]);
            const bool in = t >= lo && t < hi && (pass == 0 || (key >> pshift) == prefix);
            const uint32_t bin = in ? ((key >> shift) & ((1u << nbits) - 1)) : 0xFFFFFFFFu;
            const uint32_t peers = __match_any_sync(0xffffffffu, bin);
            if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
          }
        }
        __syncthreads();
      }
      if (pass < 2)
        find_bin<2>(hist, kk, scan_sm, &s_bin, &s_above);
      else
        find_bin<1>(hist, kk, scan_sm, &s_bin, &s_above);
      kk -= s_above;
      prefix = (prefix << nbits) | (uint32_t)s_bin;
      __syncthreads();
    }
    T = prefix;
    quota = kk;  // >= 1 keys equal to T are kept, lowest index first
  }

  // ---- ordered sweep over [0, L): sink, kept candidates, window
  uint32_t out_base = 0, tie_base = 0;
  const size_t orow = (size_t)row;
  for (int base = 0; base < L; base += 4 * kSelThreads) {
    const int t0 = base + 4 * tid;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mode == 2 && t0 < L) v = *reinterpret_cast<const float4*>(s + t0);
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t forced = 0, tie = 0;  // bit j: element t0 + j
    uint32_t nsel = 0, ntie = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + j;
      if (t >= L) continue;
      const bool cand = t >= lo && t < hi;
      bool keep = !cand;  // sink / window
      if (cand) {
        if (mode == 1) keep = true;
        if (mode == 2) {
          const uint32_t key = order_key(vv[j]);
          if (key > T) keep = true;
          else if (key == T) tie |= 1u << j;
        }
      }
      if (keep) forced |= 1u << j;
    }
    nsel = __popc(forced);
    ntie = __popc(tie);
    uint32_t total;
    const uint32_t ex = block_excl_scan<kSelThreads>(nsel | (ntie << 16), total, scan_sm);
    const uint32_t ex_sel = ex & 0xFFFFu, ex_tie = ex >> 16;
    const uint32_t tot_sel = total & 0xFFFFu, tot_tie = total >> 16;
    // ties are kept in index order while the quota lasts
    const uint32_t tie_rank0 = tie_base + ex_tie;
    uint32_t take = 0;
    if (quota > tie_rank0) take = min(quota - tie_rank0, ntie);
    uint32_t keepbits = forced;
    {
      uint32_t tb_ = tie;
      for (uint32_t n = 0; n < take; ++n) {
        keepbits |= tb_ & (~tb_ + 1u);  // lowest remaining tie
        tb_ &= tb_ - 1u;
      }
    }
    uint32_t pos = out_base + ex_sel + (min(tie_rank0, quota) - min(tie_base, quota));
    if (p.idx != nullptr) {
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (keepbits & (1u << j)) {
          if ((int)pos < p.idx_cap) p.idx[orow * p.idx_cap + pos] = t0 + j;
          ++pos;
        }
    }
    if (p.mask != nullptr) {
      uint32_t word = keepbits << ((lane & 7) * 4);
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      word |= __shfl_xor_sync(0xffffffffu, word, 2);
      word |= __shfl_xor_sync(0xffffffffu, word, 4);
      const int w = (base >> 5) + (tid >> 3);
      if ((lane & 7) == 0 && w * 32 < L) p.mask[orow * p.mask_words + w] = word;
    }
    out_base += tot_sel + (min(tie_base + tot_tie, quota) - min(tie_base, quota));
    tie_base += tot_tie;
  }
  if (tid == 0) {
    if (p.count != nullptr) p.count[orow] = (int32_t)out_base;
    const int sink_n = min(p.sink, L);
    const int win_lo = max(L - p.window, sink_n);
    const uint32_t expect = (uint32_t)(sink_n + (L - win_lo) + k);
    if (out_base != expect) atomicOr(p.status, TB_DEV_ERR_COUNT);
  }
}

}  // namespace tb
