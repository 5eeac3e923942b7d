// Prefill row selection: for every query position p of a prefill chunk and
// every query head, score the causal prefix with that position's importance
// query and keep top-k + sink + window with L -> p + 1 (model card
// "Meta-Llama-3.1-8B-Instruct-Butler", section "Method": each consumer scores
// the cached tokens with its producer's importance query, slot (l - 1) mod G,
// and keeps a top-x subset under a fixed budget plus the sink prefix and the
// local window).
//
// prefill_rows_kernel: one 1024-thread CTA per (b, h, block of 16 rows).  The
// rows share the K_imp prefix, so each K_imp row is read once per block (not
// once per row) and feeds 16 fp32 dot products, in the same dimension order
// as every other score in the library.  Scores are recomputed, not stored,
// in three passes:
//   1. first-digit (11-bit) histograms of the 16 rows' candidates;
//   2. mask words of sink, window and keys above each row's threshold bin
//      (one ballot per row and 32 tokens), and second-digit histograms of
//      the threshold bins;
//   3. keys above the 22-bit threshold prefix are OR-ed into the mask, keys
//      equal to it (a handful per row) are listed in shared memory and
//      ranked by (key desc, index asc), which also settles ties.
// A row whose 22-bit prefix holds more than kPfListCap keys (massive ties) is
// flagged; prefill_redo_kernel then recomputes it with the one-row method
// (row scores in shared memory, three radix digits, an ordered sweep).
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace tb {

constexpr int kPfRows = 16;       // rows per CTA of the blocked kernel
constexpr int kPfThreads = 1024;
constexpr int kPfListCap = 256;   // keys per row sharing the 22-bit threshold prefix
constexpr int kPfSmem = kPfRows * kHistBins * 4;

struct PrefillParams {
  const void* q_imp;   // [(B*Hq)][G][nrows][d'] kv dtype
  const float* kimp;   // [B][Hkv][max_len/256][d'][256] (kimp_index)
  uint32_t* masks;     // [B][Hq][nrows][words_per_row]
  uint32_t* status;
  uint32_t* redo;      // [B][Hq][nrows]: 1 where the blocked kernel left the row to the one-row method
  int G, slot, Hq, Hkv, max_len, row0, nrows, words_per_row;
  int keep_pct, sink, window;
};

// One row (b, h, r) by one 1024-thread CTA: the row's fp32 scores (t <= p)
// are computed once into shared memory (`srow`, p + 1 floats), the k-th
// largest order key is found by three radix digits, and an ordered sweep
// writes the row's mask words (ties at the threshold go to the lowest
// indices through a block scan).
template <typename TQ, int DIMP>
__device__ void prefill_one_row(const PrefillParams& p, int b, int h, int r, float* srow, uint32_t* hist,
                                uint32_t* scan_sm, int* s_bin_p, uint32_t* s_above_p, float* q) {
  int& s_bin = *s_bin_p;
  uint32_t& s_above = *s_above_p;
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
  __syncthreads();  // srow, hist and q are reused by the CTA's next row
}

// Persistent pass over every (b, h, row) of the call: each CTA reads the redo
// flags of its rows (strided by gridDim.x) in one parallel load, then runs the
// one-row method on the flagged ones.  Dynamic smem: `need` floats of row
// scores.
template <typename TQ, int DIMP>
__global__ void __launch_bounds__(kSelThreads, 1) prefill_redo_kernel(const PrefillParams p) {
  extern __shared__ float srow[];
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  __shared__ float q[DIMP];
  __shared__ int todo[kSelThreads];
  __shared__ int n_todo;
  const int b = blockIdx.y;
  const int per_b = p.Hq * p.nrows;
#pragma unroll 1
  for (int base = blockIdx.x; base < per_b; base += gridDim.x * kSelThreads) {
    if (threadIdx.x == 0) n_todo = 0;
    __syncthreads();
    const int i = base + threadIdx.x * gridDim.x;
    if (i < per_b && p.redo[(size_t)b * per_b + i]) todo[atomicAdd(&n_todo, 1)] = i;
    __syncthreads();
    const int n = n_todo;
    for (int j = 0; j < n; ++j) {
      const int hr = todo[j];
      prefill_one_row<TQ, DIMP>(p, b, hr / p.nrows, hr % p.nrows, srow, hist, scan_sm, &s_bin, &s_above, q);
    }
    __syncthreads();
  }
}

// The blocked method; see the file comment.  grid (ceil(nrows / 16), Hq, B).
template <typename TQ, int DIMP>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_rows_kernel(const PrefillParams p) {
  extern __shared__ __align__(16) uint32_t pf_smem[];  // hist[16][2048]; in pass 3 the key lists
  __shared__ __align__(16) float q[kPfRows][DIMP];
  __shared__ int rL[kPfRows], rhi[kPfRows], rk[kPfRows], rmode[kPfRows];
  __shared__ uint32_t rb1[kPfRows], rk1[kPfRows], rb2[kPfRows], rk2[kPfRows], rn2[kPfRows], rcnt[kPfRows];
  __shared__ uint32_t rkept[kPfRows], rabove[kPfRows], rsel[kPfRows];
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  __shared__ int s_any2;
  uint32_t* hist = pf_smem;
  uint2* lists = reinterpret_cast<uint2*>(pf_smem);  // [16][kPfListCap], pass 3 only
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gs = p.Hq / p.Hkv, g = h / gs;
  const int r0 = blockIdx.x * kPfRows;
  const int nr = min(kPfRows, p.nrows - r0);
  if (tid == 0) {
    s_any2 = 0;
    s_bin = 0;
  }
  __syncthreads();
  if (tid < kPfRows) {
    int L = 0, hi = 0, k = 0, mode = 0;
    if (tid < nr) {
      L = p.row0 + r0 + tid + 1;
      hi = L - p.window;
      const int nc = hi > p.sink ? hi - p.sink : 0;
      k = (int)min((long long)p.keep_pct * L / 100, (long long)nc);
      mode = (k > 0 && k < nc) ? 2 : (k == nc && k > 0 ? 1 : 0);
    }
    rL[tid] = L;
    rhi[tid] = hi;
    rk[tid] = k;
    rmode[tid] = mode;
    rkept[tid] = 0;
    rabove[tid] = 0;
    rsel[tid] = 0;
    rcnt[tid] = 0;
    rn2[tid] = 0;
    if (mode == 2) atomicOr(&s_any2, 1);
  }
  for (int e = tid; e < kPfRows * DIMP; e += kPfThreads) {
    const int r = e / DIMP, j = e % DIMP;
    q[r][j] = r < nr ? to_f32(reinterpret_cast<const TQ*>(p.q_imp)[((((size_t)b * p.Hq + h) * p.G + p.slot) * p.nrows +
                                                                      r0 + r) * DIMP + j])
                     : 0.f;
  }
  __syncthreads();
  const bool any2 = s_any2 != 0;
  const int Lmax = nr > 0 ? p.row0 + r0 + nr : 0;
  // rows are consecutive positions: row r's candidate range ends at hi0 + r
  const int hi0 = rhi[0];
  uint32_t m2 = 0;  // rows that take a top-k
#pragma unroll
  for (int r = 0; r < kPfRows; ++r) m2 |= (uint32_t)(rmode[r] == 2) << r;
  const size_t slab = (size_t)b * p.Hkv + g;
  // scores of token t for the 16 rows, j ascending: the same fp32 sums as every
  // other score of the library
  auto kload = [&](int t, float (&kv)[DIMP]) {
    const float* K = p.kimp + kimp_index(slab, 0, t, DIMP, p.max_len);
#pragma unroll
    for (int j = 0; j < DIMP; ++j) kv[j] = K[j * kKimpTile];
  };
  auto score_row = [&](const float (&kv)[DIMP], int r) {
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < DIMP; j += 4) {
      const float4 qq = *reinterpret_cast<const float4*>(&q[r][j]);
      acc = fmaf(qq.x, kv[j], acc);
      acc = fmaf(qq.y, kv[j + 1], acc);
      acc = fmaf(qq.z, kv[j + 2], acc);
      acc = fmaf(qq.w, kv[j + 3], acc);
    }
    return acc;
  };
  uint32_t* mbase = p.masks + (((size_t)b * p.Hq + h) * p.nrows + r0) * p.words_per_row;

  // ---- pass 1: first-digit histograms
  if (any2) {
    for (int e = tid; e < kPfRows * kHistBins; e += kPfThreads) hist[e] = 0u;
    __syncthreads();
    for (int base = 0; base < Lmax; base += kPfThreads) {
      const int t = base + tid;
      if (t < Lmax && t >= p.sink) {
        float kv[DIMP];
        kload(t, kv);
#pragma unroll 2
        for (int r = 0; r < kPfRows; ++r) {
          if (((m2 >> r) & 1u) && t < hi0 + r) {  // row r's candidates end at hi0 + r
            const float sc = score_row(kv, r);
            atomicAdd(&hist[r * kHistBins + (order_key(sc) >> 21)], 1u);
          }
        }
      }
    }
    __syncthreads();
    for (int r = 0; r < kPfRows; ++r) {
      if (rmode[r] != 2) continue;  // uniform: shared value
      find_bin<kHistBins / kPfThreads, kPfThreads>(hist + r * kHistBins, (uint32_t)rk[r], scan_sm, &s_bin, &s_above);
      if (tid == 0) {
        rb1[r] = (uint32_t)s_bin;
        rk1[r] = (uint32_t)rk[r] - s_above;
      }
      __syncthreads();
    }
    for (int e = tid; e < kPfRows * kHistBins; e += kPfThreads) hist[e] = 0u;
    __syncthreads();
  }

  // ---- pass 2: mask words (sink, window, keys above the threshold bin) and
  // second-digit histograms of the threshold bins; every word of every row
  const int nwords = p.words_per_row;
  for (int base = 0; base < nwords * 32; base += kPfThreads) {
    const int t = base + tid;
    float kv[DIMP];
    if (any2 && t < Lmax) kload(t, kv);
#pragma unroll 2
    for (int r = 0; r < kPfRows; ++r) {
      if (r >= nr) break;  // uniform
      const int L = p.row0 + r0 + r + 1;
      const bool in = t < L;
      const bool cr = t >= p.sink && t < hi0 + r;
      bool keep = in && (!cr || rmode[r] == 1);
      if (((m2 >> r) & 1u) && in && cr) {
        const uint32_t key = order_key(score_row(kv, r));
        const uint32_t d1 = key >> 21, b1 = rb1[r];
        if (d1 > b1) {
          keep = true;
        } else if (d1 == b1) {
          atomicAdd(&hist[r * kHistBins + ((key >> 10) & (kHistBins - 1))], 1u);
        }
      }
      const uint32_t word = __ballot_sync(0xffffffffu, keep);
      if (lane == 0 && (t >> 5) < nwords) {  // the last chunk may run past the row's words
        mbase[(size_t)r * nwords + (t >> 5)] = word;
        if (word) atomicAdd(&rkept[r], (uint32_t)__popc(word));
      }
    }
  }
  __syncthreads();
  if (any2) {
    for (int r = 0; r < kPfRows; ++r) {
      if (rmode[r] != 2) continue;
      find_bin<kHistBins / kPfThreads, kPfThreads>(hist + r * kHistBins, rk1[r], scan_sm, &s_bin, &s_above);
      if (tid == 0) {
        rb2[r] = (uint32_t)s_bin;
        rk2[r] = rk1[r] - s_above;
        rabove[r] = s_above;
        rn2[r] = hist[r * kHistBins + s_bin];
      }
      __syncthreads();
    }
  }
  if (tid < nr) p.redo[((size_t)b * p.Hq + h) * p.nrows + r0 + tid] = (rmode[tid] == 2 && rn2[tid] > (uint32_t)kPfListCap);
  __syncthreads();

  // ---- pass 3: keys above the 22-bit prefix into the mask, keys equal to it
  // into the row's list
  if (any2) {
    uint32_t m3 = 0;  // top-k rows this kernel finishes
#pragma unroll
    for (int r = 0; r < kPfRows; ++r) m3 |= (uint32_t)(rmode[r] == 2 && rn2[r] <= (uint32_t)kPfListCap) << r;
    for (int base = 0; base < Lmax; base += kPfThreads) {
      const int t = base + tid;
      float kv[DIMP];
      if (t < Lmax) kload(t, kv);
#pragma unroll 2
      for (int r = 0; r < kPfRows; ++r) {
        if (!((m3 >> r) & 1u)) continue;  // uniform
        bool up = false;
        if (t < Lmax && t >= p.sink && t < hi0 + r) {
          const uint32_t key = order_key(score_row(kv, r));
          if ((key >> 21) == rb1[r]) {
            const uint32_t d2 = (key >> 10) & (kHistBins - 1);
            if (d2 > rb2[r]) {
              up = true;
            } else if (d2 == rb2[r]) {
              const uint32_t pos = atomicAdd(&rcnt[r], 1u);
              if (pos < (uint32_t)kPfListCap) lists[r * kPfListCap + pos] = make_uint2(key, (uint32_t)t);
            }
          }
        }
        const uint32_t word = __ballot_sync(0xffffffffu, up);
        if (lane == 0 && word) atomicOr(&mbase[(size_t)r * nwords + (t >> 5)], word);
      }
    }
    __syncthreads();
    // rank each listed key by (key desc, index asc): the first rk2 are kept
    if (warp < nr && rmode[warp] == 2 && rn2[warp] <= (uint32_t)kPfListCap) {
      const int r = warp;
      const uint32_t n = min(rcnt[r], (uint32_t)kPfListCap);
      const uint2* lst = lists + r * kPfListCap;
      uint32_t nsel = 0;
      for (uint32_t i = lane; i < n; i += 32) {
        const uint2 e = lst[i];
        uint32_t rank = 0;
        for (uint32_t j2 = 0; j2 < n; ++j2) {
          const uint2 f = lst[j2];
          rank += (f.x > e.x) || (f.x == e.x && f.y < e.y);
        }
        if (rank < rk2[r]) {
          atomicOr(&mbase[(size_t)r * nwords + (e.y >> 5)], 1u << (e.y & 31));
          ++nsel;
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) nsel += __shfl_xor_sync(0xffffffffu, nsel, o);
      if (lane == 0) {
        rsel[r] = nsel;
        // counts: n must equal the histogram's, and kept + above + selected
        // must be sink + window + k
        const int L = rL[r];
        const int sink_n = min(p.sink, L);
        const int win_lo = max(L - p.window, sink_n);
        if (n != rn2[r] || rkept[r] + rabove[r] + nsel != (uint32_t)(sink_n + (L - win_lo) + rk[r]))
          atomicOr(p.status, TB_DEV_ERR_COUNT);
      }
    }
  }
  // rows of mode 0 / 1: the words of pass 2 are the whole set
  if (tid < nr && rmode[tid] != 2) {
    const int L = rL[tid];
    const int sink_n = min(p.sink, L);
    const int win_lo = max(L - p.window, sink_n);
    if (rkept[tid] != (uint32_t)(sink_n + (L - win_lo) + rk[tid])) atomicOr(p.status, TB_DEV_ERR_COUNT);
  }
}

}  // namespace tb
