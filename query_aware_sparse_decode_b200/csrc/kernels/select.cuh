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
// Scores are compared as monotone uint32 order keys; the k-th largest key is
// found digit by digit (11 + 11 + 10 bits).
//   hist     (standalone calls only) first-digit histogram of the candidates;
//            the decode step gets it from the score kernel instead.
//   scatter  many CTAs per row, 8192 tokens each: from the first-digit
//            histogram every CTA derives the threshold bin b1; lane = token,
//            a ballot is one mask word: sink, window and keys above b1 are
//            written to the row bitmask, keys in b1 are appended (CTA-local
//            buffer, one global atomic per CTA) to the row's candidate list.
//   resolve  one CTA per row: the candidates (a few percent of the row) are
//            loaded into shared memory, digits 2 and 3 give the k-th key T,
//            and ties at T go to the lowest indices (a radix select on the
//            index when more ties than needed); their mask bits are set.
//            Then the count check and, if asked, the ascending index list.
//   refine   (single-row selections: soft voting) many CTAs per row: when the
//            threshold bin of the first digit holds more candidates than the
//            buffer, the second digit is histogrammed over that bin, and the
//            scatter then splits the row at a 22-bit prefix instead of 11.
// A row whose threshold bin still holds more candidates than the buffer (or
// one of whose chunks overflowed its staging buffer) falls back to radix
// sweeps over the whole row and an ordered ballot/scan compaction, all inside
// the resolve CTA.
#pragma once

#include "common.cuh"
#include "reuse.cuh"

namespace tb {

constexpr int kSelThreads = 1024;   // resolve (and prefill) CTAs
constexpr int kScatThreads = 256;   // scatter / histogram CTAs
constexpr int kSelChunk = 8192;     // tokens per scatter CTA
constexpr int kSelCap = 16384;      // candidates per row
constexpr int kScatCap = 4096;      // candidates staged per scatter CTA before the global append
constexpr int kResolveSmem = kHistBins * 4 + kSelCap * 8;
constexpr int kScatSmem = kHistBins * 4 + kScatCap * 8;

struct SelectParams {
  const float* scores;    // row r of sequence b at (b * rows_per_seq + r) * row_stride
  uint32_t* hist1;        // [B*rows][2048] first-digit histograms of the candidates
  uint32_t* hist2;        // [B][2048] second-digit histograms (rows_per_seq == 1), or nullptr
  uint32_t* cand;         // [B*rows][kSelCap][2]: (key, token) of threshold-bin candidates
  uint32_t* ccount;       // [B*rows] candidates appended (zero before the scatter)
  uint32_t* kcount;       // [B*rows] tokens kept by the scatter (zero before the scatter)
  uint4* rowinfo;         // [B*rows] (prefix, rank left in it, its count, digits in the prefix)
  int32_t* idx;           // [B*rows][idx_cap] or nullptr
  int32_t* count;         // [B*rows] or nullptr
  uint32_t* mask;         // [B*rows][mask_words] (always written)
  uint32_t* status;
  long long row_stride;
  int rows_per_seq, idx_cap, mask_words;
  int keep_pct, sink, window;
  // amortised selection (decode step only; all null otherwise)
  const uint32_t* reuse;  // [B*rows] 1: this row reuses its cached selection
  const int32_t* sc_len;  // [B*rows] length of the cached selection
  uint32_t* sc_mask;      // [B*rows][mask_words] cached masks (refilled by fresh rows)
  int reuse_radius;
  int discard_scores;     // 1: the scores are a dead intermediate after the selection (dropped from L2 unwritten)
  // cluster selection (select_cluster_kernel) only
  uint32_t* ctot;         // [B*rows][2048 + 1024] the cluster's digit-2 and digit-3 totals (zero between selections)
  uint32_t* cslot;        // [B*rows][32] per-CTA tie counts (0..15) and kept counts (16..31)
  int lens[kMaxBatch];
};

// Exclusive prefix sum over a block of NT threads with one barrier: a warp
// scan, the warp totals through `sm` (>= NT / 32 words), and each warp's
// base as a reduction over the totals before it.  `sm` may be written again
// only after a later block barrier.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan_1b(uint32_t v, uint32_t& total, uint32_t* sm) {
  constexpr int NW = NT / 32;
  static_assert(NW >= 1 && NW <= 32, "1 to 32 warps");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm[warp] = x;
  __syncthreads();
  const uint32_t wt = lane < NW ? sm[lane] : 0u;
  total = __reduce_add_sync(0xffffffffu, wt);
  return __reduce_add_sync(0xffffffffu, lane < warp ? wt : 0u) + x - v;
}

// Find the bin b (scanning from the top) where the running count reaches k:
// sum(bins > b) < k <= sum(bins >= b).  NB = PER * NT bins.
template <int PER, int NT = kSelThreads>
__device__ __forceinline__ void find_bin(const uint32_t* hist, uint32_t k, uint32_t* scan_sm, int* out_bin,
                                         uint32_t* out_above) {
  constexpr int NB = PER * NT;
  const int tid = threadIdx.x;
  uint32_t c[PER];
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    c[j] = hist[NB - 1 - (tid * PER + j)];  // descending bin order
    local += c[j];
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan_1b<NT>(local, total, scan_sm);  // scan_sm is free again after the barrier below
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

// Inverse of order_key (keys of finite floats).
__device__ __forceinline__ float key_to_float(uint32_t k) {
  const uint32_t u = (k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k;
  return __uint_as_float(u);
}

struct RowShape {
  int L, lo, hi, k, mode;  // mode 0: no candidate kept, 1: all kept, 2: top-k by key
};
__device__ __forceinline__ RowShape row_shape(const SelectParams& p, int b) {
  RowShape r;
  r.L = p.lens[b];
  r.lo = p.sink;
  r.hi = r.L - p.window;
  const int nc = r.hi > r.lo ? r.hi - r.lo : 0;
  r.k = (int)min((long long)p.keep_pct * r.L / 100, (long long)nc);
  r.mode = (r.k > 0 && r.k < nc) ? 2 : (r.k == nc && r.k > 0 ? 1 : 0);
  return r;
}

// ---------------------------------------------------------------- hist
// grid (chunks, rows, B): first-digit histogram of the candidates of a chunk.
__global__ void __launch_bounds__(kScatThreads) select_hist_kernel(const SelectParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t hist[kHistBins];
  const int chunk = blockIdx.x, r = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const RowShape rs = row_shape(p, b);
  const int t_begin = chunk * kSelChunk;
  if (rs.mode != 2 || t_begin >= rs.L) return;
  const long long row = (long long)b * p.rows_per_seq + r;
  const float* s = p.scores + row * p.row_stride;
  for (int i = tid; i < kHistBins; i += kScatThreads) hist[i] = 0;
  __syncthreads();
  const int t_end = min(t_begin + kSelChunk, rs.L);
  for (int t = t_begin + tid; t < t_end; t += kScatThreads)
    if (t >= rs.lo && t < rs.hi) atomicAdd(&hist[order_key(s[t]) >> 21], 1u);
  __syncthreads();
  for (int i = tid; i < kHistBins; i += kScatThreads)
    if (hist[i]) atomicAdd(&p.hist1[row * kHistBins + i], hist[i]);
}

// ---------------------------------------------------------------- refine
// grid (chunks of kRefChunk tokens, 1, B), one row per sequence: where the
// first digit's threshold bin holds more candidates than the resolve buffer,
// histogram the second digit (bits 20..10 of the key) of the keys in that bin.
constexpr int kRefChunk = 2048;
__global__ void __launch_bounds__(kScatThreads) select_refine_kernel(const SelectParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t hist[kHistBins];
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int chunk = blockIdx.x, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31;
  const RowShape rs = row_shape(p, b);
  const int t_begin = chunk * kRefChunk;
  if (rs.mode != 2 || t_begin >= rs.hi || t_begin + kRefChunk <= rs.lo) return;
  const long long row = b;
  for (int i = tid; i < kHistBins; i += kScatThreads) hist[i] = p.hist1[row * kHistBins + i];
  __syncthreads();
  find_bin<kHistBins / kScatThreads, kScatThreads>(hist, (uint32_t)rs.k, scan_sm, &s_bin, &s_above);
  const uint32_t b1 = (uint32_t)s_bin;
  if (hist[b1] <= (uint32_t)kSelCap) return;  // the same decision in every thread
  __syncthreads();
  for (int i = tid; i < kHistBins; i += kScatThreads) hist[i] = 0;
  __syncthreads();
  const float* s = p.scores + row * p.row_stride;
  const int t_end = min(t_begin + kRefChunk, rs.hi);
  for (int base = t_begin; base < t_end; base += kScatThreads) {  // warp-uniform bounds
    const int t = base + tid;
    bool in = false;
    uint32_t bin = 0xFFFFFFFFu;
    if (t >= rs.lo && t < t_end) {
      const uint32_t key = order_key(s[t]);
      in = (key >> 21) == b1;
      if (in) bin = (key >> 10) & (kHistBins - 1);
    }
    const uint32_t peers = __match_any_sync(0xffffffffu, bin);
    if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
  }
  __syncthreads();
  for (int i = tid; i < kHistBins; i += kScatThreads)
    if (hist[i]) atomicAdd(&p.hist2[row * kHistBins + i], hist[i]);
}

// ---------------------------------------------------------------- scatter
// grid (chunks, rows, B), 256 threads: warp w owns tokens [w*1024, w*1024+1024)
// of the CTA's chunk, all loaded up front (8 float4 per lane).  The CTA's
// kept-token count goes to a per-row counter that the resolve kernel checks.
__global__ void __launch_bounds__(kScatThreads, 4) select_scatter_kernel(const SelectParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint32_t scat_smem[];
  uint32_t* hist = scat_smem;               // [2048]
  uint32_t* lkey = hist + kHistBins;        // [kScatCap]
  uint32_t* lidx = lkey + kScatCap;         // [kScatCap]
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_n, s_base, s_kept;
  const int chunk = blockIdx.x, r = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const RowShape rs = row_shape(p, b);
  const int t_begin = chunk * kSelChunk;
  if (t_begin >= rs.L) return;
  const long long row = (long long)b * p.rows_per_seq + r;
  if (p.reuse != nullptr && p.reuse[row]) {
    // the row reuses its cached selection: cached top-k (widened by the
    // radius) inside the current candidates, plus the current sink and window
    const uint32_t* cm = p.sc_mask + row * p.mask_words;
    const int hi_prev = p.sc_len[row] - p.window, lo = p.sink;
    auto topk = [&](int w) -> uint32_t {
      return (w < 0 || w >= p.mask_words) ? 0u : (cm[w] & range_bits(w * 32, lo, hi_prev));
    };
    uint32_t kept = 0;
    const int w_end = min((t_begin + kSelChunk) >> 5, (rs.L + 31) >> 5);
    for (int w = (t_begin >> 5) + tid; w < w_end; w += kScatThreads) {
      uint32_t x = topk(w);
      if (p.reuse_radius > 0) {
        const uint32_t prev = topk(w - 1), next = topk(w + 1);
        const uint64_t below = ((uint64_t)x << 32) | prev;  // tokens 32(w-1) .. 32w+31
        const uint64_t above = ((uint64_t)next << 32) | x;  // tokens 32w .. 32(w+1)+31
        uint32_t d = x;
        for (int sft = 1; sft <= p.reuse_radius; ++sft)
          d |= (uint32_t)(below >> (32 - sft)) | (uint32_t)(above >> sft);
        x = d;
      }
      const uint32_t word = (x & range_bits(w * 32, lo, rs.hi)) | range_bits(w * 32, 0, min(p.sink, rs.L)) |
                            range_bits(w * 32, max(rs.L - p.window, 0), rs.L);
      p.mask[row * p.mask_words + w] = word;
      kept += __popc(word);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
    if (lane == 0 && kept) atomicAdd(&p.kcount[row], kept);
    return;
  }
  const float* s = p.scores + row * p.row_stride;
  // the chunk's scores are requested first, so their latency overlaps the
  // threshold search below.  A warp step covers 256 tokens: lane owns 8
  // consecutive tokens (two float4), lanes 4m..4m+3 form mask word m
  constexpr int STEPS = 4;
  const int wt0 = t_begin + warp * 1024;
  float4 v[STEPS][2];
#pragma unroll
  for (int u = 0; u < STEPS; ++u) {
    const int t0 = wt0 + u * 256 + 8 * lane;
#pragma unroll
    for (int h = 0; h < 2; ++h)
      v[u][h] = (rs.mode == 2 && t0 + 4 * h < rs.L) ? *reinterpret_cast<const float4*>(s + t0 + 4 * h)
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float f_lo = 0.f, f_hi = 0.f;
  bool hi_open = false;
  bool collect = false;  // candidates are gathered only when the resolve buffer can hold the bin
  if (tid == 0) {
    s_n = 0;
    s_kept = 0;
  }
  if (rs.mode == 2) {
    for (int i = tid; i < kHistBins; i += kScatThreads) hist[i] = p.hist1[row * kHistBins + i];
    __syncthreads();
    find_bin<kHistBins / kScatThreads, kScatThreads>(hist, (uint32_t)rs.k, scan_sm, &s_bin, &s_above);
    uint32_t prefix = (uint32_t)s_bin, kleft = (uint32_t)rs.k - s_above, nbin = hist[s_bin];
    int shift = 21;
    if (p.hist2 != nullptr && nbin > (uint32_t)kSelCap) {  // split the bin by the second digit
      __syncthreads();
      for (int i = tid; i < kHistBins; i += kScatThreads) hist[i] = p.hist2[(size_t)b * kHistBins + i];
      __syncthreads();
      find_bin<kHistBins / kScatThreads, kScatThreads>(hist, kleft, scan_sm, &s_bin, &s_above);
      prefix = (prefix << 11) | (uint32_t)s_bin;
      kleft -= s_above;
      nbin = hist[s_bin];
      shift = 10;
    }
    f_lo = key_to_float(prefix << shift);          // smallest key of the threshold bin
    f_hi = key_to_float((prefix + 1u) << shift);   // smallest key above it
    hi_open = prefix == (0xFFFFFFFFu >> shift);
    collect = nbin <= (uint32_t)kSelCap;
    if (chunk == 0 && tid == 0)  // the resolve CTA reads the row's prefix from here
      p.rowinfo[row] = make_uint4(prefix, kleft, nbin, shift == 21 ? 1u : 2u);
  } else {
    __syncthreads();
  }
  uint32_t kept = 0;  // tokens of the words this lane stores
#pragma unroll
  for (int u = 0; u < STEPS; ++u) {
    const int tw = wt0 + u * 256;
    if (tw >= rs.L) break;  // warp-uniform
    const int t0 = tw + 8 * lane;
    const float vv[8] = {v[u][0].x, v[u][0].y, v[u][0].z, v[u][0].w, v[u][1].x, v[u][1].y, v[u][1].z, v[u][1].w};
    uint32_t keep = 0, cbits = 0;
    if (rs.mode == 2 && tw >= rs.lo && tw + 256 <= rs.hi) {
      // interior step: every token is an in-range candidate
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        keep |= (uint32_t)(vv[j] >= f_hi) << j;
        cbits |= (uint32_t)(vv[j] >= f_lo) << j;
      }
      if (hi_open) keep = 0;
      cbits &= ~keep;
    } else {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int t = t0 + j;
        const bool in = t < rs.L;
        const bool cand = t >= rs.lo && t < rs.hi;
        bool kp = in && (!cand || rs.mode == 1);
        bool c = false;
        if (rs.mode == 2 && in && cand) {
          const bool above = !hi_open && vv[j] >= f_hi;
          kp = above;
          c = !above && vv[j] >= f_lo;
        }
        keep |= (uint32_t)kp << j;
        cbits |= (uint32_t)c << j;
      }
    }
    uint32_t word = keep << ((lane & 3) * 8);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if ((lane & 3) == 0 && t0 < rs.L) {
      p.mask[row * p.mask_words + (t0 >> 5)] = word;
      kept += __popc(word);
    }
    if (!collect) cbits = 0;
    if (__any_sync(0xffffffffu, cbits != 0)) {
      const uint32_t cnt = __popc(cbits);
      uint32_t x = cnt;  // inclusive prefix over the lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      uint32_t base = 0;
      if (lane == 31) base = atomicAdd(&s_n, x);
      base = __shfl_sync(0xffffffffu, base, 31);
      uint32_t pos = base + x - cnt;
      while (cbits) {
        const int j = __ffs(cbits) - 1;
        cbits &= cbits - 1u;
        if (pos < (uint32_t)kScatCap) {
          lkey[pos] = order_key(vv[j]);
          lidx[pos] = (uint32_t)(t0 + j);
        }
        ++pos;
      }
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) kept += __shfl_xor_sync(0xffffffffu, kept, o);
  if (lane == 0 && kept) atomicAdd(&s_kept, kept);
  __syncthreads();
  if (tid == 0 && s_kept) atomicAdd(&p.kcount[row], s_kept);
  if (rs.mode != 2 || !collect) return;
  const uint32_t n = min(s_n, (uint32_t)kScatCap);
  if (tid == 0) {
    s_base = atomicAdd(&p.ccount[row], s_n);
    // this chunk held more of the bin than its staging buffer: the list is
    // incomplete, so the resolve CTA takes the whole-row path for this row
    if (s_n > (uint32_t)kScatCap) atomicOr(&p.ccount[row], 0x80000000u);
  }
  __syncthreads();
  uint32_t* dst = p.cand + (size_t)row * kSelCap * 2;
  for (uint32_t i = tid; i < n; i += kScatThreads) {
    const uint32_t pos = s_base + i;
    if (pos < (uint32_t)kSelCap) *reinterpret_cast<uint2*>(dst + 2 * pos) = make_uint2(lkey[i], lidx[i]);
  }
}

// ---------------------------------------------------------------- resolve
// Radix select of the `k` largest among the eligible entries of a shared
// array, one digit at a time (digits of 11, 11 and 10 bits over a 32-bit
// key), from pass `first_pass` with `prefix` the digits already fixed.
// Warp-aggregated shared atomics keep heavily repeated keys cheap.
template <class Key>
__device__ __forceinline__ void smem_radix(int n, Key key_of, int first_pass, uint32_t prefix, uint32_t k,
                                           uint32_t* hist, uint32_t* scan_sm, int* s_bin, uint32_t* s_above,
                                           uint32_t& T, uint32_t& quota) {
  const int tid = threadIdx.x, lane = tid & 31;
  uint32_t kk = k;
#pragma unroll 1
  for (int pass = first_pass; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nbits = pass == 2 ? 10 : 11;
    const int pshift = pass == 1 ? 21 : 10;
    for (int i = tid; i < kHistBins; i += kSelThreads) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kSelThreads) {
      const int i = base + tid;
      bool in = false;
      uint32_t key = 0;
      if (i < n) in = key_of(i, key);
      in = in && (pass == 0 || (key >> pshift) == prefix);
      const uint32_t bin = in ? ((key >> shift) & ((1u << nbits) - 1)) : 0xFFFFFFFFu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
    }
    __syncthreads();
    if (pass < 2)
      find_bin<2>(hist, kk, scan_sm, s_bin, s_above);
    else
      find_bin<1>(hist, kk, scan_sm, s_bin, s_above);
    kk -= *s_above;
    prefix = (prefix << nbits) | (uint32_t)*s_bin;
    __syncthreads();
  }
  T = prefix;
  quota = kk;
}

// The resolve CTA of a row is the last reader of its histograms and candidate
// counter: it clears them for the next selection (so no separate zeroing pass
// precedes the next score kernel).
__device__ __forceinline__ void clear_row_state(const SelectParams& p, long long row, int b) {
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) p.hist1[row * kHistBins + i] = 0u;
  if (p.hist2 != nullptr)
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) p.hist2[(size_t)b * kHistBins + i] = 0u;
  if (threadIdx.x == 0) {
    p.ccount[row] = 0u;
    p.kcount[row] = 0u;
  }
}

__global__ void __launch_bounds__(kSelThreads, 1) select_resolve_kernel(const SelectParams p) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(16) uint32_t res_smem[];
  uint32_t* hist = res_smem;            // [2048]
  uint32_t* ckey = hist + kHistBins;    // [kSelCap]
  uint32_t* cidx = ckey + kSelCap;      // [kSelCap]
  __shared__ uint32_t scan_sm[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int r = blockIdx.x, b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const RowShape rs = row_shape(p, b);
  const int L = rs.L, lo = rs.lo, hi = rs.hi, k = rs.k;
  const long long row = (long long)b * p.rows_per_seq + r;
  const bool reused = p.reuse != nullptr && p.reuse[row] != 0u;
  const int mode = reused ? 0 : rs.mode;  // a reused row's mask is complete after the scatter
  const size_t orow = (size_t)row;
  const float* s = p.scores + row * p.row_stride;
  const int lwords = (L + 31) >> 5;
  // a fresh selection of a row with a selection cache refills it below
  const bool refill = p.reuse != nullptr && !reused && rs.mode == 2;

  bool fallback = false;
  uint32_t prefix1 = 0, k1 = 0, n1 = 0;
  int next_pass = 1;  // digits already fixed by the scatter: 1 or 2
  if (mode == 2) {
    const uint4 info = p.rowinfo[row];
    prefix1 = info.x;
    k1 = info.y;
    n1 = info.z;
    next_pass = info.w == 2u ? 2 : 1;
    fallback = n1 > (uint32_t)kSelCap;
  }

  if (mode == 2 && !fallback) fallback = (p.ccount[row] >> 31) != 0u;  // a staging buffer overflowed
  if (!fallback) {
    if (mode == 2) {
      uint32_t n = p.ccount[row];
      if (n != n1) {  // histogram and scores disagree: flag it, stay in bounds
        if (tid == 0) atomicOr(p.status, TB_DEV_ERR_COUNT);
        n = min(n, (uint32_t)kSelCap);
      }
      const uint32_t* src = p.cand + orow * kSelCap * 2;
      for (uint32_t i = tid; i < n; i += kSelThreads) {
        const uint2 e = *reinterpret_cast<const uint2*>(src + 2 * i);
        ckey[i] = e.x;
        cidx[i] = e.y;
      }
      __syncthreads();
      uint32_t T, quota;
      smem_radix(
          (int)n,
          [&](int i, uint32_t& key) {
            key = ckey[i];
            return true;
          },
          next_pass, prefix1, k1, hist, scan_sm, &s_bin, &s_above, T, quota);
      // ties at T: keep the `quota` lowest indices
      uint32_t ntie_local = 0;
      for (uint32_t i = tid; i < n; i += kSelThreads) ntie_local += ckey[i] == T;
      uint32_t ntie;
      (void)block_excl_scan<kSelThreads>(ntie_local, ntie, scan_sm);
      uint32_t J = 0;  // threshold on ~index among the ties when only some of them are kept
      const bool all_ties = ntie == quota;
      if (!all_ties) {
        uint32_t q2;
        smem_radix(
            (int)n,
            [&](int i, uint32_t& key) {
              key = ~cidx[i];
              return ckey[i] == T;
            },
            0, 0u, quota, hist, scan_sm, &s_bin, &s_above, J, q2);
      }
      for (uint32_t i = tid; i < n; i += kSelThreads) {
        const uint32_t key = ckey[i], t = cidx[i];
        if (key > T || (key == T && (all_ties || ~t >= J)))
          atomicOr(&p.mask[orow * p.mask_words + (t >> 5)], 1u << (t & 31));
      }
      __threadfence_block();
      __syncthreads();
    }
    // ---- count check and optional ascending index list.  Without a list the
    // count is the scatter's kept tokens plus the k1 candidates marked here
    // (exactly k1 by construction); with one, the mask is read back.
    uint32_t total = 0;
    if (p.idx != nullptr) {
      const int per = (lwords + kSelThreads - 1) / kSelThreads;
      const int w0 = min(lwords, tid * per), w1 = min(lwords, w0 + per);
      uint32_t mine = 0;
      for (int w = w0; w < w1; ++w) mine += __popc(__ldcg(p.mask + orow * p.mask_words + w));
      uint32_t pos = block_excl_scan<kSelThreads>(mine, total, scan_sm);
      for (int w = w0; w < w1; ++w) {
        uint32_t m = __ldcg(p.mask + orow * p.mask_words + w);
        while (m) {
          const int j = __ffs(m) - 1;
          m &= m - 1u;
          if ((int)pos < p.idx_cap) p.idx[orow * p.idx_cap + pos] = w * 32 + j;
          ++pos;
        }
      }
    } else {
      total = p.kcount[row] + (mode == 2 ? k1 : 0u);
    }
    if (tid == 0) {
      if (p.count != nullptr) p.count[orow] = (int32_t)total;
      const int sink_n = min(p.sink, L);
      const int win_lo = max(L - p.window, sink_n);
      // a reused set has the cached top-k's size, not this step's k
      if (!reused && total != (uint32_t)(sink_n + (L - win_lo) + k)) atomicOr(p.status, TB_DEV_ERR_COUNT);
    }
    if (refill)
      for (int w = tid; w < lwords; w += kSelThreads) p.sc_mask[orow * p.mask_words + w] = __ldcg(p.mask + orow * p.mask_words + w);
    __syncthreads();  // every thread has read the counters before they are cleared
    clear_row_state(p, row, b);
    return;
  }

  // ================================================================ fallback
  uint32_t T, quota;
  {
    uint32_t prefix = prefix1, kk = k1;
#pragma unroll 1
    for (int pass = next_pass; pass < 3; ++pass) {
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
    if (t0 < L) v = *reinterpret_cast<const float4*>(s + t0);
    const float vv[4] = {v.x, v.y, v.z, v.w};
    uint32_t forced = 0, tie = 0;  // bit j: element t0 + j
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int t = t0 + j;
      if (t >= L) continue;
      const bool cand = t >= lo && t < hi;
      bool keep = !cand;  // sink / window
      if (cand) {
        const uint32_t key = order_key(vv[j]);
        if (key > T) keep = true;
        else if (key == T) tie |= 1u << j;
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
    uint32_t word = keepbits << ((lane & 7) * 4);
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    word |= __shfl_xor_sync(0xffffffffu, word, 4);
    const int w = (base >> 5) + (tid >> 3);
    if ((lane & 7) == 0 && w < lwords) p.mask[orow * p.mask_words + w] = word;
    out_base += tot_sel + (min(tie_base + tot_tie, quota) - min(tie_base, quota));
    tie_base += tot_tie;
  }
  if (tid == 0) {
    if (p.count != nullptr) p.count[orow] = (int32_t)out_base;
    const int sink_n = min(p.sink, L);
    const int win_lo = max(L - p.window, sink_n);
    if (out_base != (uint32_t)(sink_n + (L - win_lo) + k)) atomicOr(p.status, TB_DEV_ERR_COUNT);
  }
  if (refill) {
    __syncthreads();  // the mask words written above
    for (int w = tid; w < lwords; w += kSelThreads) p.sc_mask[orow * p.mask_words + w] = __ldcg(p.mask + orow * p.mask_words + w);
  }
  clear_row_state(p, row, b);
}

}  // namespace tb
