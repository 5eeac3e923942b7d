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
// One 1024-thread CTA per row; scores are read as monotone uint32 order keys.
// Fast path (one ordered sweep of the row):
//   1. first-digit histogram (top 11 key bits) of the candidates - from the
//      score kernel, else built here - gives the threshold bin b1 and how
//      many keys lie above it;
//   2. the sweep sets, in a shared-memory copy of the row bitmask, every
//      token surely kept (sink, window, digit > b1) and appends the
//      candidates of bin b1, in index order (block scan), to a shared buffer;
//   3. the remaining two digits are resolved on that buffer only; ties at the
//      final key go to the lowest indices (the buffer is in index order);
//   4. the bitmask, the count and optionally the ascending index list are
//      written out from shared memory.
// Fallback (bin b1 larger than the buffer, or rows beyond the shared bitmask):
// three radix sweeps over the row with warp-aggregated histograms, then an
// ordered ballot/scan compaction.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kSelThreads = 1024;
constexpr int kSelCap = 16384;       // candidate buffer entries (key + index)
constexpr int kSelMaskWords = 8192;  // shared bitmask words: rows up to 262144 tokens
constexpr int kSelSmemBytes = kHistBins * 4 + kSelCap * 8 + kSelMaskWords * 4;

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

// Inverse of order_key (for keys of finite floats).
__device__ __forceinline__ float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__global__ void __launch_bounds__(kSelThreads, 1) select_kernel(const SelectParams p) {
  extern __shared__ __align__(16) uint32_t sel_smem[];
  uint32_t* hist = sel_smem;                           // [2048]
  uint32_t* ckey = hist + kHistBins;                   // [kSelCap]
  uint32_t* cidx = ckey + kSelCap;                     // [kSelCap]
  uint32_t* smask = cidx + kSelCap;                    // [kSelMaskWords]
  __shared__ uint32_t scan_sm[32];
  __shared__ uint2 scan2_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const int r = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int L = p.lens[b];
  const long long row = (long long)b * p.rows_per_seq + r;
  const float* s = p.scores + row * p.row_stride;
  const int lo = p.sink, hi = L - p.window;
  const int nc = hi > lo ? hi - lo : 0;
  const int k = (int)min((long long)p.keep_pct * L / 100, (long long)nc);
  const int lwords = (L + 31) >> 5;
  const size_t orow = (size_t)row;

  int mode = 0;  // 0: no candidate kept, 1: all kept, 2: threshold + quota ties
  if (k == nc && k > 0) mode = 1;
  if (k > 0 && k < nc) mode = 2;

  // ---- first digit: histogram of the candidates' top 11 key bits
  int b1 = 0;
  uint32_t k1 = 0, n1 = 0;
  if (mode == 2) {
    if (p.hist1 != nullptr) {
      for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = p.hist1[row * kHistBins + i];
    } else {
      for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int base = lo & ~3; base < hi; base += 4 * kSelThreads) {
        const int t0 = base + 4 * tid;
        if (t0 < hi) {
          const float4 v = *reinterpret_cast<const float4*>(s + t0);
          const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int j = 0; j < 4; ++j)
            if (t0 + j >= lo && t0 + j < hi) atomicAdd(&hist[order_key(vv[j]) >> 21], 1u);
        }
      }
    }
    __syncthreads();
    find_bin<2>(hist, (uint32_t)k, scan_sm, &s_bin, &s_above);
    b1 = s_bin;
    k1 = (uint32_t)k - s_above;
    n1 = hist[b1];
    __syncthreads();
  }
  const bool fast = lwords <= kSelMaskWords && (mode != 2 || n1 <= (uint32_t)kSelCap);

  uint32_t T = 0, quota = 0;
  if (fast) {
    // ---- one ordered sweep: sure bits into the shared mask, bin-b1 candidates
    // into the buffer.  Lane = token: an iteration covers STEPS x 1024 tokens,
    // step j of warp w holds tokens base + j*1024 + w*32 + lane, so a ballot
    // is one mask word.  The threshold-bin test is two float compares against
    // the bin's boundary values (the key map is monotone; -0.0 == +0.0 holds
    // for both).  Candidates keep index order through a (step, warp) prefix.
    constexpr int STEPS = 16;
    constexpr int ITER = STEPS * kSelThreads;
    const int warp = tid >> 5;
    const float f_lo = key_to_float((uint32_t)b1 << 21);         // smallest key of bin b1
    const float f_hi = key_to_float(((uint32_t)b1 + 1u) << 21);  // smallest key above bin b1
    const bool hi_open = b1 == (int)(kHistBins - 1);             // no key lies above the top bin
    uint32_t nbuf = 0;
    uint32_t* wcnt = hist;  // [STEPS][32] candidate counts per (step, warp); hist is free during the sweep
    for (int base = 0; base < L; base += ITER) {
      float v[STEPS];
#pragma unroll
      for (int j = 0; j < STEPS; ++j) {
        const int t = base + j * kSelThreads + tid;
        v[j] = (mode == 2 && t < L) ? s[t] : 0.f;
      }
      uint32_t cmask[STEPS];
#pragma unroll
      for (int j = 0; j < STEPS; ++j) {
        const int t = base + j * kSelThreads + tid;
        const bool in = t < L;
        const bool cand = t >= lo && t < hi;
        bool keep = in && (!cand || mode == 1);
        bool c = false;
        if (mode == 2 && in && cand) {
          const bool above = !hi_open && v[j] >= f_hi;
          keep = above;
          c = !above && v[j] >= f_lo;
        }
        const uint32_t word = __ballot_sync(0xffffffffu, keep);
        const int w = (base + j * kSelThreads) / 32 + warp;
        if (lane == 0 && w < lwords) smask[w] = word;
        cmask[j] = __ballot_sync(0xffffffffu, c);
      }
      if (mode == 2) {
        __syncthreads();  // previous users of wcnt are done
        if (lane < STEPS) {
          uint32_t cnt = 0;
#pragma unroll
          for (int j = 0; j < STEPS; ++j) cnt = j == lane ? __popc(cmask[j]) : cnt;
          wcnt[lane * 32 + warp] = cnt;
        }
        __syncthreads();
        if (warp < STEPS) {  // warp j: exclusive prefix over the 32 warps of step j
          const uint32_t c = wcnt[warp * 32 + lane];
          uint32_t x = c;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
          }
          wcnt[warp * 32 + lane] = x - c;
          if (lane == 31) scan_sm[warp] = x;  // step total
        }
        __syncthreads();
        uint32_t step_base[STEPS];
        uint32_t run = nbuf;
#pragma unroll
        for (int j = 0; j < STEPS; ++j) {
          step_base[j] = run;
          run += scan_sm[j];
        }
#pragma unroll
        for (int j = 0; j < STEPS; ++j) {
          if (cmask[j] & (1u << lane)) {
            const uint32_t pos = step_base[j] + wcnt[j * 32 + warp] + __popc(cmask[j] & lanemask_lt());
            if (pos < (uint32_t)kSelCap) {
              ckey[pos] = order_key(v[j]);
              cidx[pos] = (uint32_t)(base + j * kSelThreads + tid);
            }
          }
        }
        nbuf = run;
      }
    }
    __syncthreads();
    if (mode == 2 && nbuf != n1) {  // histogram and scores disagree: flag it, stay in bounds
      if (tid == 0) atomicOr(p.status, TB_DEV_ERR_COUNT);
      nbuf = min(nbuf, (uint32_t)kSelCap);
    }

    if (mode == 2) {
      // ---- digits 2 and 3 on the buffer
      uint32_t prefix = (uint32_t)b1, kk = k1;
#pragma unroll 1
      for (int pass = 1; pass < 3; ++pass) {
        const int shift = pass == 1 ? 10 : 0;
        const int nbits = pass == 1 ? 11 : 10;
        const int pshift = pass == 1 ? 21 : 10;
        for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = 0;
        __syncthreads();
        for (int i = tid; i < (int)nbuf; i += kSelThreads) {
          const uint32_t key = ckey[i];
          if ((key >> pshift) == prefix) atomicAdd(&hist[(key >> shift) & ((1u << nbits) - 1)], 1u);
        }
        __syncthreads();
        if (pass == 1)
          find_bin<2>(hist, kk, scan_sm, &s_bin, &s_above);
        else
          find_bin<1>(hist, kk, scan_sm, &s_bin, &s_above);
        kk -= s_above;
        prefix = (prefix << nbits) | (uint32_t)s_bin;
        __syncthreads();
      }
      T = prefix;
      quota = kk;
      // ---- keys above T, and the first `quota` ties in index (= buffer) order
      uint32_t tie_base = 0;
      for (int base = 0; base < (int)nbuf; base += kSelThreads) {
        const int i = base + tid;
        const uint32_t key = i < (int)nbuf ? ckey[i] : 0u;
        const bool tie = i < (int)nbuf && key == T;
        uint32_t total;
        const uint32_t rank = tie_base + block_excl_scan<kSelThreads>(tie ? 1u : 0u, total, scan_sm);
        if (i < (int)nbuf && (key > T || (tie && rank < quota))) {
          const uint32_t t = cidx[i];
          atomicOr(&smask[t >> 5], 1u << (t & 31));
        }
        tie_base += total;
      }
      __syncthreads();
    }

    // ---- write out: mask, count, ascending index list
    uint32_t cnt_local = 0;
    for (int w = tid; w < lwords; w += kSelThreads) {
      const uint32_t m = smask[w];
      if (p.mask != nullptr) p.mask[orow * p.mask_words + w] = m;
      cnt_local += __popc(m);
    }
    uint32_t total_cnt;
    (void)block_excl_scan<kSelThreads>(cnt_local, total_cnt, scan_sm);
    if (p.idx != nullptr) {
      // thread owns consecutive words [w0, w1)
      const int per = (lwords + kSelThreads - 1) / kSelThreads;
      const int w0 = min(lwords, tid * per), w1 = min(lwords, w0 + per);
      uint32_t mine = 0;
      for (int w = w0; w < w1; ++w) mine += __popc(smask[w]);
      uint32_t tot;
      uint32_t pos = block_excl_scan<kSelThreads>(mine, tot, scan_sm);
      for (int w = w0; w < w1; ++w) {
        uint32_t m = smask[w];
        while (m) {
          const int j = __ffs(m) - 1;
          m &= m - 1u;
          if ((int)pos < p.idx_cap) p.idx[orow * p.idx_cap + pos] = w * 32 + j;
          ++pos;
        }
      }
    }
    if (tid == 0) {
      if (p.count != nullptr) p.count[orow] = (int32_t)total_cnt;
      const int sink_n = min(p.sink, L);
      const int win_lo = max(L - p.window, sink_n);
      if (total_cnt != (uint32_t)(sink_n + (L - win_lo) + k)) atomicOr(p.status, TB_DEV_ERR_COUNT);
    }
    return;
  }

  // ================================================================ fallback
  if (mode == 2) {
    uint32_t prefix = (uint32_t)b1, kk = k1;
#pragma unroll 1
    for (int pass = 1; pass < 3; ++pass) {
      const int shift = pass == 1 ? 10 : 0;
      const int nbits = pass == 1 ? 11 : 10;
      const int pshift = pass == 1 ? 21 : 10;
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
          const bool in = t >= lo && t < hi && (key >> pshift) == prefix;
          if (!__any_sync(0xffffffffu, in)) continue;
          const uint32_t bin = in ? ((key >> shift) & ((1u << nbits) - 1)) : 0xFFFFFFFFu;
          const uint32_t peers = __match_any_sync(0xffffffffu, bin);
          if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
        }
      }
      __syncthreads();
      if (pass == 1)
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
  for (int base = 0; base < L; base += 4 * kSelThreads) {
    const int t0 = base + 4 * tid;
    float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
    if (mode == 2 && t0 < L) v = *reinterpret_cast<const float4*>(s + t0);
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t forced = 0, tie = 0;  // bit j: element t0 + j
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
    const uint32_t nsel = __popc(forced), ntie = __popc(tie);
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
