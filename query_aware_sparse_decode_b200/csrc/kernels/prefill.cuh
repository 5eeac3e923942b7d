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
// in two passes, and a third pass works on what the second kept:
//   1. first-digit (11-bit) histograms of the 16 rows' candidates;
//   2. mask words of sink, window and keys above each row's threshold bin
//      (one ballot per row and 32 tokens), second-digit histograms of the
//      threshold bins, and each row's keys of its threshold bin listed in
//      shared memory, up to kPfBinCap per row;
//   3. from those lists, keys above the 22-bit threshold prefix are OR-ed
//      into the mask and keys equal to it (a handful per row) are listed and
//      ranked by (key desc, index asc), which also settles ties.  Rows whose
//      bin did not fit recompute their tiles for this pass instead.
// Tiles whose 32 tokens are candidates of all 16 rows skip the per-token
// range checks.
// A row whose 22-bit prefix holds more than kPfListCap keys (massive ties) is
// flagged; prefill_redo_kernel then recomputes it with the one-row method
// (row scores in shared memory, three radix digits, an ordered sweep).
#pragma once

#include "common.cuh"
#include "select.cuh"

namespace tb {

constexpr int kPfRows = 16;       // rows per CTA of the blocked kernel
constexpr int kPfThreads = 512;
constexpr int kPfListCap = 256;   // keys per row sharing the 22-bit threshold prefix
// Prefixes the prefill selection accepts: the one-row method keeps a row's
// fp32 scores in 200 KB of shared memory.  Below 65536 tokens, so a 16-bit
// counter holds any bin's count.
constexpr int kPfMaxPrefix = 200 * 1024 / 4;
static_assert(kPfMaxPrefix < 65536, "16-bit second-digit counters");
// Pass 2 keeps each row's keys of its threshold bin in shared memory (with
// 16-bit second-digit counters, two per word) so that pass 3 works on those
// lists instead of recomputing the tiles: up to kPfBinCap keys per row.
constexpr int kPfBinCap = 1280;
constexpr int kPfHist16Words = kPfRows * kHistBins / 2;
constexpr int kPfSmem = kPfHist16Words * 4 + kPfRows * kPfBinCap * 8;  // >= the 32-bit first-digit histograms
static_assert(kPfSmem >= kPfRows * kHistBins * 4, "pass 1 histograms fit");

struct PrefillParams {
  const void* q_imp;   // [(B*Hq)][G][nrows][d'] kv dtype
  const void* kimp;    // [B][Hkv][max_len/256][d'][256] (kimp_index), KT elements
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
template <typename TQ, typename KT, int DIMP>
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
    const KT* K = reinterpret_cast<const KT*>(p.kimp) + kimp_index(slab, 0, t, DIMP, p.max_len);
    float acc = 0.f;
#pragma unroll
    for (int j = 0; j < DIMP; ++j) acc = fmaf(q[j], to_f32(K[j * kKimpTile]), acc);
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
template <typename TQ, typename KT, int DIMP>
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
      prefill_one_row<TQ, KT, DIMP>(p, b, hr / p.nrows, hr % p.nrows, srow, hist, scan_sm, &s_bin, &s_above, q);
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------- blocked
// TF32 helpers for the score tiles.  A bf16 importance query is exact in TF32.
// A K_imp value v is carried as hi + lo: hi is v cut to TF32 width and lo the
// exact remainder v - hi, of which the tensor core reads a TF32-width head.
// Together they keep at least 21 of v's 24 significand bits, so a tile score
// differs from the fp32 dot product by about 1e-6 relative: far inside the
// selection's tie band.  Every pass recomputes the same tiles the same way.
__device__ __forceinline__ uint32_t to_tf32(float x) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;\n" : "=r"(r) : "f"(x));
  return r;
}
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = to_tf32(x);
  lo = to_tf32(x - __uint_as_float(hi));
}
// D += A (16x8, row) * B (8x8, col), TF32 in, fp32 accumulate
__device__ __forceinline__ void mma_tf32_1688(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// find_bin for one row by one warp: lane l sums bins 2047 - 64 l - j
// (j = 0..63; read in a lane-skewed order, so no two lanes hit one bank),
// a warp scan gives each lane the count above its range, and the lane whose
// range holds the k-th key walks it from the top.  PACKED: 16-bit counters,
// two per word (bin 2w in the low half of word w).  bin = -1 when the
// histogram holds fewer than k keys.
template <bool PACKED>
__device__ __forceinline__ void warp_find_bin(const uint32_t* hist, uint32_t k, int& bin, uint32_t& above) {
  const int lane = threadIdx.x & 31;
  auto count = [&](int b) -> uint32_t {
    return PACKED ? (hist[b >> 1] >> ((b & 1) << 4)) & 0xFFFFu : hist[b];
  };
  uint32_t local = 0;
#pragma unroll 8
  for (int j = 0; j < 64; ++j) local += count(kHistBins - 1 - (64 * lane + ((j + lane) & 63)));
  uint32_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t excl = incl - local;
  const uint32_t holder = __ballot_sync(0xffffffffu, excl < k && k <= incl);
  int fb = -1;
  uint32_t fa = 0;
  if (holder != 0u && lane == __ffs(holder) - 1) {
    uint32_t run = excl;
    for (int j = 0; j < 64; ++j) {
      const int b = kHistBins - 1 - (64 * lane + j);
      const uint32_t c = count(b);
      if (run + c >= k) {
        fb = b;
        fa = run;
        break;
      }
      run += c;
    }
  }
  const int src = holder != 0u ? __ffs(holder) - 1 : 0;
  bin = __shfl_sync(0xffffffffu, fb, src);
  above = __shfl_sync(0xffffffffu, fa, src);
}

// The blocked method; see the file comment.  grid (ceil(nrows / 16), Hq, B),
// 1024 threads.  The 16 rows are the M dimension of mma.sync m16n8k8 TF32
// tiles: a warp takes 32 tokens at a time (four n-tiles of 8; one mask word
// per row), and lane (g, c) = (lane / 4, lane % 4) holds the scores of rows g
// and g + 8 for tokens 2c and 2c + 1 of each n-tile.
template <typename TQ, typename KT, int DIMP>
__global__ void __launch_bounds__(kPfThreads, 1) prefill_rows_kernel(const PrefillParams p) {
  constexpr int KS = DIMP / 8;                        // k-steps of 8 dimensions
  constexpr bool QSPLIT = sizeof(TQ) == 4;            // fp32 queries need hi + lo too
  constexpr bool KBF16 = sizeof(KT) == 2;             // bf16 K_imp: exact in TF32
  // pass 1: hist[16][2048]; pass 2: 16-bit counters [16][1024] words + bin lists
  // [16][kPfBinCap] (or 32-bit hist[16][2048] for long rows); pass 3: lists [16][kPfListCap]
  extern __shared__ __align__(16) uint32_t pf_smem[];
  __shared__ int rmode[kPfRows], rk[kPfRows];
  __shared__ uint32_t rb1[kPfRows], rk1[kPfRows], rb2[kPfRows], rk2[kPfRows], rn2[kPfRows], rcnt[kPfRows];
  __shared__ uint32_t rbin[kPfRows];  // keys of the threshold bin appended per row (pass 2)
  __shared__ uint32_t rkept[kPfRows], rabove[kPfRows];
  __shared__ int s_any2, s_not2, s_big2;
  uint32_t* hist = pf_smem;
  uint2* lists = reinterpret_cast<uint2*>(pf_smem);  // [16][kPfListCap], pass 3 only
  uint2* blists = reinterpret_cast<uint2*>(pf_smem + kPfHist16Words);  // [16][kPfBinCap], passes 2-3
  const int h = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, cq = lane & 3;
  const int gs = p.Hq / p.Hkv, g = h / gs;
  const int r0 = blockIdx.x * kPfRows;
  const int nr = min(kPfRows, p.nrows - r0);
  if (tid == 0) {
    s_any2 = 0;
    s_not2 = 0;
    s_big2 = 0;
  }
  __syncthreads();
  if (tid < kPfRows) {
    int k = 0, mode = 0;
    if (tid < nr) {
      const int L = p.row0 + r0 + tid + 1;
      const int hi = L - p.window;
      const int nc = hi > p.sink ? hi - p.sink : 0;
      k = (int)min((long long)p.keep_pct * L / 100, (long long)nc);
      mode = (k > 0 && k < nc) ? 2 : (k == nc && k > 0 ? 1 : 0);
    }
    rk[tid] = k;
    rmode[tid] = mode;
    rkept[tid] = 0;
    rabove[tid] = 0;
    rcnt[tid] = 0;
    rbin[tid] = 0;
    rn2[tid] = 0;
    rb1[tid] = 0;
    rb2[tid] = 0;
    if (mode == 2) atomicOr(&s_any2, 1);
    if (mode != 2) atomicOr(&s_not2, 1);
  }
  __syncthreads();
  const bool any2 = s_any2 != 0;
  // every one of the 16 rows resolves a top-k (no short or padding rows):
  // interior tiles then need no per-token range or mode checks
  const bool all2 = s_not2 == 0;
  const int Lmax = nr > 0 ? p.row0 + r0 + nr : 0;
  const int L0 = p.row0 + r0 + 1;        // row r covers tokens [0, L0 + r)
  const int hi0 = L0 - p.window;         // row r's candidates are [sink, hi0 + r)
  const size_t slab = (size_t)b * p.Hkv + g;
  // A fragments (the 16 rows' importance queries), constant for the kernel
  uint32_t afr[KS][4], afl[KS][4];
  {
    const TQ* qi = reinterpret_cast<const TQ*>(p.q_imp);
    auto qv = [&](int r, int j) -> float {
      return r < nr ? to_f32(qi[((((size_t)b * p.Hq + h) * p.G + p.slot) * p.nrows + r0 + r) * DIMP + j]) : 0.f;
    };
#pragma unroll
    for (int ks = 0; ks < KS; ++ks) {
      const float v[4] = {qv(gq, ks * 8 + cq), qv(gq + 8, ks * 8 + cq), qv(gq, ks * 8 + cq + 4),
                          qv(gq + 8, ks * 8 + cq + 4)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        if (QSPLIT) {
          split_tf32(v[e], afr[ks][e], afl[ks][e]);
        } else {
          afr[ks][e] = __float_as_uint(v[e]);  // exact
          afl[ks][e] = 0u;
        }
      }
    }
  }
  // scores of the 16 rows for the 32 tokens [t0, t0 + 32): sc[n][i], n-tile n,
  // i = (row gq, token 2cq), (gq, 2cq+1), (gq+8, 2cq), (gq+8, 2cq+1)
  // The B operands of a tile: the K_imp values this lane feeds to the four
  // n-tiles (token t0 + 8 n + gq, dimensions ks * 8 + cq and + 4), all
  // requested before the first mma of the tile.
  using TileK = float[4][KS][2];
  auto tile_load = [&](int t0, TileK& kv) {
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const int t = t0 + 8 * n + gq;
      const bool ok = t < Lmax;
      const KT* K = reinterpret_cast<const KT*>(p.kimp) + kimp_index(slab, 0, ok ? t : 0, DIMP, p.max_len);
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        kv[n][ks][0] = ok ? to_f32(K[(ks * 8 + cq) * kKimpTile]) : 0.f;
        kv[n][ks][1] = ok ? to_f32(K[(ks * 8 + cq + 4) * kKimpTile]) : 0.f;
      }
    }
  };
  auto tile_mma = [&](const TileK& kv, float (&sc)[4][4]) {
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        const float k0 = kv[n][ks][0];
        const float k1 = kv[n][ks][1];
        // hi: the value cut to TF32 width; lo: the exact fp32 remainder, of
        // which the tensor core reads the TF32-width head.  A bf16 K_imp has
        // 8 significant bits, so it is exact in TF32 and has no remainder.
        const uint32_t h0 = __float_as_uint(k0) & 0xFFFFE000u, h1 = __float_as_uint(k1) & 0xFFFFE000u;
        mma_tf32_1688(sc[n], afr[ks], h0, h1);
        if (!KBF16) {
          const uint32_t l0 = __float_as_uint(k0 - __uint_as_float(h0));
          const uint32_t l1 = __float_as_uint(k1 - __uint_as_float(h1));
          mma_tf32_1688(sc[n], afr[ks], l0, l1);
        }
        if (QSPLIT) mma_tf32_1688(sc[n], afl[ks], h0, h1);
      }
    }
  };
  auto tile_scores = [&](int t0, float (&sc)[4][4]) {
    TileK kv;
    tile_load(t0, kv);
    tile_mma(kv, sc);
  };

  uint32_t* mbase = p.masks + (((size_t)b * p.Hq + h) * p.nrows + r0) * p.words_per_row;
  const int nwords = p.words_per_row;
  const int nsteps = (Lmax + 31) / 32;
  const int ra = gq, rb = gq + 8;  // this lane's rows
  // value i of n-tile n: row (i < 2 ? ra : rb), token t0 + 8 n + 2 cq + (i & 1)

  // ---- pass 1: first-digit histograms
  if (any2) {
    for (int e = tid; e < kPfRows * kHistBins; e += kPfThreads) hist[e] = 0u;
    __syncthreads();
    const bool m2a = rmode[ra] == 2, m2b = rmode[rb] == 2;
    for (int ws = warp; ws < nsteps; ws += kPfThreads / 32) {
      const int t0 = ws * 32;
      float sc[4][4];
      tile_scores(t0, sc);
      if (all2 && t0 >= p.sink && t0 + 32 <= hi0) {  // every token a candidate of every row (warp-uniform)
#pragma unroll
        for (int n = 0; n < 4; ++n)
#pragma unroll
          for (int i = 0; i < 4; ++i)
            atomicAdd(&hist[(i < 2 ? ra : rb) * kHistBins + (order_key(sc[n][i]) >> 21)], 1u);
        continue;
      }
#pragma unroll
      for (int n = 0; n < 4; ++n) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = i < 2 ? ra : rb;
          const bool m2 = i < 2 ? m2a : m2b;
          const int t = t0 + 8 * n + 2 * cq + (i & 1);
          if (m2 && t >= p.sink && t < hi0 + row)
            atomicAdd(&hist[row * kHistBins + (order_key(sc[n][i]) >> 21)], 1u);
        }
      }
    }
    __syncthreads();
    static_assert(kPfThreads / 32 >= kPfRows, "a warp per row");
    if (warp < kPfRows && rmode[warp] == 2) {  // the 16 rows' threshold bins at once
      int bin;
      uint32_t ab;
      warp_find_bin<false>(hist + warp * kHistBins, (uint32_t)rk[warp], bin, ab);
      if (lane == 0) {
        if (bin < 0) {  // inconsistent scores: count error, indices kept in bounds
          atomicOr(p.status, TB_DEV_ERR_COUNT);
          bin = 0;
          ab = 0;
        }
        rb1[warp] = (uint32_t)bin;
        rk1[warp] = (uint32_t)rk[warp] - ab;
      }
    }
    __syncthreads();
    for (int e = tid; e < kPfRows * kHistBins; e += kPfThreads) hist[e] = 0u;
    __syncthreads();
  }

  // ---- pass 2: every mask word of every row (sink, window, keys above the
  // threshold bin), second-digit histograms of the threshold bins (16-bit
  // counters), and the threshold bin's keys listed per row
  auto member = [&](int row, uint32_t key, int t) {
    const uint32_t d2 = (key >> 10) & (kHistBins - 1);
    atomicAdd(&hist[row * (kHistBins / 2) + (d2 >> 1)], 1u << ((d2 & 1u) << 4));
    const uint32_t slot = atomicAdd(&rbin[row], 1u);
    if (slot < (uint32_t)kPfBinCap) blists[row * kPfBinCap + slot] = make_uint2(key, (uint32_t)t);
  };
  {
    const int mda = rmode[ra], mdb = rmode[rb];
    const uint32_t b1a = rb1[ra], b1b = rb1[rb];
    for (int ws = warp; ws < nwords; ws += kPfThreads / 32) {
      const int t0 = ws * 32;
      float sc[4][4] = {};
      if (any2 && t0 < Lmax) tile_scores(t0, sc);  // warp-uniform
      uint32_t wa = 0, wb = 0;
      if (all2 && t0 >= p.sink && t0 + 32 <= hi0) {  // every token a candidate of every row (warp-uniform)
#pragma unroll
        for (int n = 0; n < 4; ++n) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int pos = 8 * n + 2 * cq + (i & 1);
            const uint32_t key = order_key(sc[n][i]);
            const uint32_t d1 = key >> 21, b1 = i < 2 ? b1a : b1b;
            if (d1 > b1) {
              if (i < 2) wa |= 1u << pos;
              else wb |= 1u << pos;
            } else if (d1 == b1) {
              member(i < 2 ? ra : rb, key, t0 + pos);
            }
          }
        }
      } else {
#pragma unroll
      for (int n = 0; n < 4; ++n) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = i < 2 ? ra : rb, md = i < 2 ? mda : mdb;
          const int pos = 8 * n + 2 * cq + (i & 1);
          const int t = t0 + pos;
          const bool in = t < L0 + row;
          const bool cr = t >= p.sink && t < hi0 + row;
          bool keep = in && (!cr || md == 1);
          if (md == 2 && in && cr) {
            const uint32_t key = order_key(sc[n][i]);
            const uint32_t d1 = key >> 21, b1 = i < 2 ? b1a : b1b;
            if (d1 > b1) {
              keep = true;
            } else if (d1 == b1) {
              member(row, key, t);
            }
          }
          if (keep) {
            if (i < 2) wa |= 1u << pos;
            else wb |= 1u << pos;
          }
        }
      }
      }
      wa |= __shfl_xor_sync(0xffffffffu, wa, 1);
      wa |= __shfl_xor_sync(0xffffffffu, wa, 2);
      wb |= __shfl_xor_sync(0xffffffffu, wb, 1);
      wb |= __shfl_xor_sync(0xffffffffu, wb, 2);
      if (cq == 0) {
        if (ra < nr) {
          mbase[(size_t)ra * nwords + ws] = wa;
          if (wa) atomicAdd(&rkept[ra], (uint32_t)__popc(wa));
        }
        if (rb < nr) {
          mbase[(size_t)rb * nwords + ws] = wb;
          if (wb) atomicAdd(&rkept[rb], (uint32_t)__popc(wb));
        }
      }
    }
  }
  __syncthreads();
  if (any2) {
    if (warp < kPfRows && rmode[warp] == 2) {
      const int r = warp;
      int bin;
      uint32_t ab;
      warp_find_bin<true>(hist + r * (kHistBins / 2), rk1[r], bin, ab);
      if (lane == 0) {
        if (bin < 0) {
          atomicOr(p.status, TB_DEV_ERR_COUNT);
          bin = 0;
          ab = 0;
        }
        rb2[r] = (uint32_t)bin;
        rk2[r] = rk1[r] - ab;
        rabove[r] = ab;
        rn2[r] = (hist[r * (kHistBins / 2) + (bin >> 1)] >> ((bin & 1) << 4)) & 0xFFFFu;
      }
    }
    __syncthreads();
  }
  if (tid < nr) p.redo[((size_t)b * p.Hq + h) * p.nrows + r0 + tid] = (rmode[tid] == 2 && rn2[tid] > (uint32_t)kPfListCap);
  if (tid < kPfRows && rmode[tid] == 2 && rn2[tid] > (uint32_t)kPfListCap) atomicOr(&s_big2, 1);
  __syncthreads();

  // ---- pass 3: keys above the 22-bit prefix into the mask, keys equal to it
  // into the row's list
  if (any2) {
    // a row is resolved from its bin list when the list holds the whole bin
    auto listed = [&](int r) { return rbin[r] <= (uint32_t)kPfBinCap; };
    {  // keys of the listed rows' bins above the 22-bit prefix into the mask, keys at it into the row's list
      for (int e = tid; e < kPfRows * kPfBinCap; e += kPfThreads) {
        const int r = e / kPfBinCap, i = e % kPfBinCap;
        if (rmode[r] != 2 || rn2[r] > (uint32_t)kPfListCap || !listed(r) || (uint32_t)i >= rbin[r]) continue;
        const uint2 x = blists[e];
        const uint32_t d2 = (x.x >> 10) & (kHistBins - 1);
        if (d2 > rb2[r]) {
          atomicOr(&mbase[(size_t)r * nwords + (x.y >> 5)], 1u << (x.y & 31));
        } else if (d2 == rb2[r]) {
          const uint32_t slot = atomicAdd(&rcnt[r], 1u);
          if (slot < (uint32_t)kPfListCap) lists[r * kPfListCap + slot] = x;
        }
      }
    }
    const bool m3a = rmode[ra] == 2 && rn2[ra] <= (uint32_t)kPfListCap && !listed(ra);
    const bool m3b = rmode[rb] == 2 && rn2[rb] <= (uint32_t)kPfListCap && !listed(rb);
    const uint32_t b1a = rb1[ra], b1b = rb1[rb], b2a = rb2[ra], b2b = rb2[rb];
    const bool all3 = all2 && __all_sync(0xffffffffu, m3a && m3b) && s_big2 == 0;
    const bool any3 = __syncthreads_or(m3a || m3b);  // some row is left to the tile recompute
    for (int ws = warp; any3 && ws < nsteps; ws += kPfThreads / 32) {
      const int t0 = ws * 32;
      float sc[4][4];
      tile_scores(t0, sc);
      uint32_t ua = 0, ub = 0;
      // every token a candidate of every row, every row listed (warp-uniform)
      const bool inner = all3 && t0 >= p.sink && t0 + 32 <= hi0;
#pragma unroll
      for (int n = 0; n < 4; ++n) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int row = i < 2 ? ra : rb;
          const bool m3 = i < 2 ? m3a : m3b;
          const int pos = 8 * n + 2 * cq + (i & 1);
          const int t = t0 + pos;
          if (!inner && (!m3 || t < p.sink || t >= hi0 + row)) continue;
          const uint32_t key = order_key(sc[n][i]);
          if ((key >> 21) != (i < 2 ? b1a : b1b)) continue;
          const uint32_t d2 = (key >> 10) & (kHistBins - 1), b2 = i < 2 ? b2a : b2b;
          if (d2 > b2) {
            if (i < 2) ua |= 1u << pos;
            else ub |= 1u << pos;
          } else if (d2 == b2) {
            const uint32_t slot = atomicAdd(&rcnt[row], 1u);
            if (slot < (uint32_t)kPfListCap) lists[row * kPfListCap + slot] = make_uint2(key, (uint32_t)t);
          }
        }
      }
      ua |= __shfl_xor_sync(0xffffffffu, ua, 1);
      ua |= __shfl_xor_sync(0xffffffffu, ua, 2);
      ub |= __shfl_xor_sync(0xffffffffu, ub, 1);
      ub |= __shfl_xor_sync(0xffffffffu, ub, 2);
      if (cq == 0) {
        if (ua) atomicOr(&mbase[(size_t)ra * nwords + ws], ua);
        if (ub) atomicOr(&mbase[(size_t)rb * nwords + ws], ub);
      }
    }
    __syncthreads();
    // rank each listed key by (key desc, index asc): the first rk2 are kept
    for (int r = warp; r < nr; r += kPfThreads / 32) {
      if (rmode[r] != 2 || rn2[r] > (uint32_t)kPfListCap) continue;
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
        // n must equal the histogram's count, and kept + above + selected
        // must be sink + window + k
        const int L = L0 + r;
        const int sink_n = min(p.sink, L);
        const int win_lo = max(L - p.window, sink_n);
        if (n != rn2[r] || rkept[r] + rabove[r] + nsel != (uint32_t)(sink_n + (L - win_lo) + rk[r]))
          atomicOr(p.status, TB_DEV_ERR_COUNT);
      }
    }
  }
  // rows of mode 0 / 1: the words of pass 2 are the whole set
  if (tid < nr && rmode[tid] != 2) {
    const int L = L0 + tid;
    const int sink_n = min(p.sink, L);
    const int win_lo = max(L - p.window, sink_n);
    if (rkept[tid] != (uint32_t)(sink_n + (L - win_lo) + rk[tid])) atomicOr(p.status, TB_DEV_ERR_COUNT);
  }
}

}  // namespace tb
