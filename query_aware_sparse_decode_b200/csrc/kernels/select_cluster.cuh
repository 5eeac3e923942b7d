// butler_topk + butler_merge in one launch: the selection of a row by a
// thread-block cluster (model card "Meta-Llama-3.1-8B-Instruct-Butler",
// section "Method": top-x subset under a fixed token budget plus a sink
// prefix and a recent local window; section "Memory requirements":
// fixed_<N>pc, min_sparse_index, sliding_window).
//
//   k = floor(P * L / 100), candidates C = [sink, L - window),
//   Sel = [0, min(sink, L)) U top_min(k, |C|)(C) U [max(L - window, 0), L),
//   order (score desc, index asc), -0.0 == +0.0.
//
// A cluster of NC CTAs (NC in 1..16) owns one row; CTA c owns the tokens
// [c * chunk, (c + 1) * chunk).  Scores are compared as monotone uint32 order
// keys and the k-th largest key T is found digit by digit (11 + 11 + 10
// bits).  The row's scores are read from L2 once:
//   1. digit 1 comes from the first-digit histogram that the score kernel
//      (or select_hist_kernel) built; every CTA finds the threshold bin b1
//      while its first score loads are in flight.
//   2. one pass over the CTA's tokens (16-byte loads, batches of four per
//      thread double-buffered in registers; scores compared as floats with
//      the bin's bounds) writes, per 32-token word, "kept for sure" (sink,
//      window, keys above bin b1) into a shared copy of the CTA's mask words,
//      and appends the scores of bin b1 (a few percent of the row) to a
//      shared list; after the pass the list's scores become keys and their
//      second digit is histogrammed (a convergent loop over the list).
//   3. in a cluster of two, after a cluster barrier each CTA adds the other
//      CTA's digit-2 histogram from its shared memory (distributed shared
//      memory) to its own; in larger clusters each CTA adds its histogram
//      into the row's total in L2 (atomics) and reads the total back after a
//      cluster barrier.  Digit 2, then digit 3 over the list through L2, give
//      T and the number `quota` of keys equal to T that are kept.
//   4. ties at T go to the lowest indices.  When every key equal to T is
//      kept (the usual case) each CTA keeps its own; otherwise each CTA posts
//      its count, and after a barrier CTA c keeps the first
//      clamp(quota - (ties on CTAs < c), 0, its ties) of its own, found by an
//      ordered scan over a shared tie bitmap.
//   5. list keys above T and the kept ties are OR-ed into the shared mask
//      words, which are written once.  The kept counts are added up in L2;
//      the last CTA to finish (a ticket counter) checks the total, writes the
//      optional count and clears the row's first-digit histogram and totals,
//      so the next selection needs no zeroing pass.  With an index list the
//      counts are posted per CTA instead and a barrier gives every CTA its
//      offset.
// The cluster barriers (barrier.cluster arrive/release, wait/acquire) are the
// only waits between CTAs; in a cluster of two the digit-2 histogram is read
// from the other CTA's shared memory (the digit-3 barrier keeps it alive
// until both have read), everything else goes through L2; no CTA waits on a
// flag.  A CTA whose list overflows re-reads its tokens from
// L2 for steps 3-5 instead; the result is the same.  Rows that keep none or
// all of their candidates, and rows reusing a cached selection, write their
// words directly.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "reuse.cuh"
#include "select.cuh"

namespace tb {

// Threads per CTA: 512 (two CTAs per SM) when the rows' clusters need more
// than one CTA per SM, 1024 (one per SM) when they fit one wave of one CTA
// per SM (few rows: every SM then runs one 32-warp CTA)
constexpr int kClThreadsMany = 512;
constexpr int kClThreadsFew = 1024;
constexpr int kClChunkMax = 65536;            // tokens per CTA
constexpr int kClWordsMax = kClChunkMax / 32;  // mask words per CTA
constexpr int kClListCap = 4096;              // keys of the threshold bin kept in shared memory
constexpr int kClMaxCluster = 16;
constexpr int kClHist3 = 1024;                // bins of the 10-bit last digit
constexpr int kClBatch = 4;                   // 16-byte loads per thread and batch of the first pass
constexpr int kClTotWords = kHistBins + kClHist3 + 2;  // per row in ctot: totals, kept count, CTA ticket
static_assert(kClTotWords % 2 == 0 && (kHistBins + kClHist3) % 2 == 0, "the (kept count, ticket) pair is one 8-byte word");
constexpr int kClSlotWords = 2 * kClMaxCluster;    // per row in cslot

struct ClusterSelectSmem {
  uint32_t mword[kClWordsMax];      // the CTA's mask words
  uint32_t tbits[kClWordsMax];      // keys equal to T among the CTA's tokens
  uint2 list[kClListCap];           // (key, token - c0) of the threshold bin's keys
  uint32_t hist[kHistBins];         // this CTA's digit-2 histogram (read by the cluster's other CTAs)
  uint32_t hist3[kClHist3];         // this CTA's digit-3 histogram
  uint32_t scan[32];
  uint32_t n_list, pre_ties, ntie_all, last, kept_total;
  int bin;
  uint32_t above, bin_count;
};
constexpr int kClSmem = ((int)sizeof(ClusterSelectSmem) + 15) / 16 * 16;
// Dynamic shared memory of an NT-thread CTA: the struct, then the first
// pass's staging area (float4 [kClBatch][NT]: a lane's batch of scores, read
// back by the lane itself for its threshold-bin members).
template <int NT>
constexpr int cl_smem() { return kClSmem + kClBatch * NT * 16; }

// Host: cluster size and chunk of a selection over rows of at most maxL
// tokens, `nrows` rows in all.  max_active[i] is how many clusters of 2^i
// CTAs (1..16) can be resident at once (0: not launchable).  Among the sizes
// whose CTAs cover a row (nc * kClChunkMax >= L): the largest that keeps all
// rows' clusters resident in one wave, with at most about four CTAs per SM
// and at least 256 tokens per CTA; else the smallest covering size that is
// resident in one wave; else the smallest covering size.  Returns false when
// no size covers the row.
inline bool cluster_select_shape(int num_sms, long long nrows, int maxL, const int (&max_active)[5], int* nc_out,
                                 int* chunk_out) {
  const long long L = maxL > 1 ? maxL : 1;
  int pick = 0, one_wave = 0, cover = 0;
  for (int i = 0; i < 5; ++i) {
    const int nc = 1 << i;
    if (max_active[i] < 1 || (long long)nc * kClChunkMax < L) continue;
    if (!cover) cover = nc;
    if (nrows > max_active[i]) continue;
    if (!one_wave) one_wave = nc;
    if (nrows * nc <= 4LL * num_sms && (L + nc - 1) / nc >= 256) pick = nc;
  }
  const int nc = pick ? pick : (one_wave ? one_wave : cover);
  if (!nc) return false;
  const long long chunk = ((L + nc - 1) / nc + 255) / 256 * 256;
  *nc_out = nc;
  *chunk_out = (int)chunk;
  return chunk <= kClChunkMax;
}

// Host: launch with programmatic stream serialization and a cluster of
// `nc` CTAs along x.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      int nc, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = nc;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The bin b where the running count from the top of an NB-bin histogram
// reaches k (sum(bins > b) < k <= sum(bins >= b)), from the counts the
// threads hold: thread t holds bins NB - 1 - (t * PER + j), j = 0..PER-1
// (descending), so that no staging through shared memory is needed.  One
// scan barrier and one closing barrier.  Also gives the bin's count.  A
// histogram holding fewer than k keys (inconsistent scores, e.g. NaN)
// records TB_DEV_ERR_COUNT and yields bin 0, so every index stays in bounds.
template <int NT, int PER>
__device__ __forceinline__ uint32_t find_bin_held(const uint32_t (&c)[PER], uint32_t k, ClusterSelectSmem& sm,
                                                  uint32_t* status, uint32_t& above, uint32_t& count) {
  constexpr int NB = PER * NT;
  const int tid = threadIdx.x;
  uint32_t local = 0;
#pragma unroll
  for (int j = 0; j < PER; ++j) local += c[j];
  if (tid == 0) sm.bin = -1;  // before the scan's barrier; the crossing thread writes after it
  uint32_t total;
  const uint32_t excl = block_excl_scan_1b<NT>(local, total, sm.scan);
  if (excl < k && k <= excl + local) {
    uint32_t run = excl;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
      if (run + c[j] >= k) {
        sm.bin = NB - 1 - (tid * PER + j);
        sm.above = run;
        sm.bin_count = c[j];
        break;
      }
      run += c[j];
    }
  }
  __syncthreads();
  const int bin = sm.bin;
  if (bin < 0) {
    if (tid == 0) atomicOr(status, TB_DEV_ERR_COUNT);
    above = 0;
    count = 0;
    return 0u;
  }
  above = sm.above;
  count = sm.bin_count;
  return (uint32_t)bin;
}

// This thread's bins of an NB-word histogram in L2 (NB = PER * NT), in the
// order find_bin_held wants: bins NB - 1 - (t * PER + j).
template <int NT, int PER>
__device__ __forceinline__ void load_bins_desc(const uint32_t* h, uint32_t (&c)[PER]) {
  constexpr int NB = PER * NT;
  const uint32_t* lo = h + NB - (threadIdx.x + 1) * PER;  // this thread's bins, ascending
  if constexpr (PER == 4) {
    const uint4 x = __ldcg(reinterpret_cast<const uint4*>(lo));
    c[0] = x.w; c[1] = x.z; c[2] = x.y; c[3] = x.x;
  } else if constexpr (PER == 2) {
    const uint2 x = __ldcg(reinterpret_cast<const uint2*>(lo));
    c[0] = x.y; c[1] = x.x;
  } else {
#pragma unroll
    for (int j = 0; j < PER; ++j) c[j] = __ldcg(lo + PER - 1 - j);
  }
}

// Adds this CTA's histogram into the row's total in L2 (non-empty bins only).
template <int NT, int NB>
__device__ __forceinline__ void hist_to_total(const uint32_t* hist, uint32_t* total) {
  for (int i = threadIdx.x; i < NB; i += NT) {
    const uint32_t v = hist[i];
    if (v) atomicAdd(total + i, v);
  }
}

// Calls f(t, key) for every candidate token t of [a, b) (a a multiple of 4,
// candidates [lo, hi)), reading the scores with four 16-byte loads per
// thread in flight.  The row holds max_len >= b scores, a multiple of 256,
// so every 16-byte load that starts below b stays inside the row.
template <int NT, class F>
__device__ __forceinline__ void visit_candidates(const float* srow, int a, int b, int lo, int hi, F f) {
  const int start = max(a, lo) & ~3, end = min(b, hi);
  for (int base = start; base < end; base += 16 * NT) {
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t0 = base + 4 * (threadIdx.x + NT * u);
      v[u] = t0 < end ? __ldcg(reinterpret_cast<const float4*>(srow + t0)) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t0 = base + 4 * (threadIdx.x + NT * u);
      const float vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int t = t0 + j;
        if (t >= lo && t < end) f(t, order_key(vv[j]));
      }
    }
  }
}

// grid (NC, rows, B), cluster (NC, 1, 1), NT threads, kClSmem bytes.
template <int NT>
__global__ void __launch_bounds__(NT, 1024 / NT) select_cluster_kernel(const SelectParams p, int chunk) {
  constexpr int kClThreads = NT;
  constexpr int kClWarps = NT / 32;
  pdl_wait();
  pdl_trigger();
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint8_t cl_raw[];
  ClusterSelectSmem& sm = *reinterpret_cast<ClusterSelectSmem*>(cl_raw);
  float4* stage = reinterpret_cast<float4*>(cl_raw + kClSmem);  // [kClBatch][NT]
  const int nc = (int)cluster.num_blocks();
  const int c = (int)cluster.block_rank();
  const int r = blockIdx.y, b = blockIdx.z, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const RowShape rs = row_shape(p, b);
  const long long row = (long long)b * p.rows_per_seq + r;
  const int c0 = c * chunk;                    // a multiple of 256: word-aligned
  const int c1 = min(c0 + chunk, rs.L);
  const int nw = c1 > c0 ? (c1 - c0 + 31) >> 5 : 0;  // this CTA's words holding tokens < L
  const bool reused = p.reuse != nullptr && p.reuse[row] != 0u;
  const bool topk = rs.mode == 2 && !reused;
  const float* srow = p.scores + row * p.row_stride;
  uint32_t* tot = p.ctot + row * kClTotWords;   // [2048] digit-2 total, then [1024] digit-3 total
  uint32_t* slot = p.cslot + row * kClSlotWords;  // [16] tie counts, [16] kept counts

  if (topk) {
    for (int i = tid; i < nw; i += kClThreads) sm.tbits[i] = 0u;
    for (int i = tid; i < kHistBins; i += kClThreads) sm.hist[i] = 0u;
    for (int i = tid; i < kClHist3; i += kClThreads) sm.hist3[i] = 0u;
    if (tid == 0) sm.n_list = 0u;
    // Warp w owns words [wb, we) and walks them in batches of 16 words: lane l
    // loads the 16 bytes at tokens 32 * (w0 + 4u + l / 8) + 4 * (l % 8),
    // u = 0..3, so lane group l / 8 holds word w0 + 4u + l / 8.  The next
    // batch's loads are in flight while this one is processed (two register
    // batches).
    const int wpw = (nw + kClWarps - 1) / kClWarps;
    const int wb = min(warp * wpw, nw), we = min(wb + wpw, nw);
    float4 va[kClBatch], vb[kClBatch];
    auto load_batch = [&](float4 (&v)[kClBatch], int w0) {
#pragma unroll
      for (int u = 0; u < kClBatch; ++u) {
        const int w = w0 + 4 * u + (lane >> 3);
        const int tv = c0 + 32 * w + 4 * (lane & 7);
        v[u] = (w < we && tv < c1) ? __ldcg(reinterpret_cast<const float4*>(srow + tv))
                                   : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    };
    // ---- digit 1 from the row's first-digit histogram; the bin's bounds as floats.
    // The histogram is requested first, then the first batch of scores, whose
    // latency overlaps the digit-1 search.
    constexpr int P1 = kHistBins / NT;
    uint32_t h1[P1];
    load_bins_desc<NT, P1>(p.hist1 + row * kHistBins, h1);
    if (wb < we) load_batch(va, wb);
    uint32_t above, bcount;
    const uint32_t b1 = find_bin_held<NT, P1>(h1, (uint32_t)rs.k, sm, p.status, above, bcount);
    const uint32_t kleft = (uint32_t)rs.k - above;
    const bool hi_open = b1 == (uint32_t)(kHistBins - 1);                   // no key above the bin
    const float f_lo = key_to_float(b1 << 21);                              // smallest key of the bin
    // smallest key above it; NaN when there is none (no score compares >= NaN)
    const float f_hi = hi_open ? __int_as_float(0x7fc00000) : key_to_float((b1 + 1u) << 21);
    // ---- one pass over the CTA's tokens: sure-keep words and the bin's scores.
    // Float comparisons against the bin's bounds decide the same as the keys
    // (the key map is monotone and folds -0.0 onto +0.0, as IEEE comparison
    // does).  A lane's bin members of a batch (bit 4u + j: its load u,
    // element j) are appended with one warp scan and one shared atomic; a
    // lane with members stages its batch in shared memory and reads back
    // only those.
    static_assert(kClBatch == 4, "the word exchange below assumes four loads per batch");
    auto process = [&](const float4 (&v)[kClBatch], int w0) {
      const bool interior =
          w0 + 4 * kClBatch <= we && c0 + 32 * w0 >= rs.lo && c0 + 32 * (w0 + 4 * kClBatch) <= min(rs.hi, c1);
      const int p8 = lane & 7;
      uint32_t kx[kClBatch];  // load u's sure-keep nibble at bits 4 * p8 of its word
      uint32_t memb = 0;     // bit 4u + j
#pragma unroll
      for (int u = 0; u < kClBatch; ++u) {
        const float vv[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        uint32_t keep = 0, mb = 0;
        if (interior) {  // every token a valid candidate
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            keep |= (uint32_t)(vv[j] >= f_hi) << j;
            mb |= (uint32_t)(vv[j] >= f_lo) << j;
          }
          mb &= ~keep;
        } else {
          const int w = w0 + 4 * u + (lane >> 3);
          const int tv = c0 + 32 * w + 4 * p8;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int t = tv + j;
            const bool valid = w < we && t < c1;
            const bool cand = t >= rs.lo && t < rs.hi;
            const bool up = vv[j] >= f_hi;
            keep |= (uint32_t)(valid && (!cand || up)) << j;
            mb |= (uint32_t)(valid && cand && !up && vv[j] >= f_lo) << j;
          }
        }
        kx[u] = keep << (4 * p8);
        memb |= mb << (4 * u);
      }
      // Each 8-lane group's four words, OR-ed over the group in three
      // exchange rounds: over lane bit 2 a lane keeps two words and sends
      // two, over bit 1 it keeps one and sends one, over bit 0 both lanes
      // complete the same word.  Lane p8 ends with word u = 2 * (p8 >> 2 & 1)
      // + (p8 >> 1 & 1); the even lane stores it.
      const bool hb = (p8 & 4) != 0, mbit = (p8 & 2) != 0;
      uint32_t k0 = hb ? kx[2] : kx[0], k1 = hb ? kx[3] : kx[1];
      const uint32_t s0 = hb ? kx[0] : kx[2], s1 = hb ? kx[1] : kx[3];
      k0 |= __shfl_xor_sync(0xffffffffu, s0, 4);
      k1 |= __shfl_xor_sync(0xffffffffu, s1, 4);
      uint32_t word = mbit ? k1 : k0;
      word |= __shfl_xor_sync(0xffffffffu, mbit ? k0 : k1, 2);
      word |= __shfl_xor_sync(0xffffffffu, word, 1);
      const int wq = w0 + 4 * ((hb ? 2 : 0) + (mbit ? 1 : 0)) + (lane >> 3);
      if ((p8 & 1) == 0 && wq < we) sm.mword[wq] = word;
      if (!__any_sync(0xffffffffu, memb != 0u)) return;
      if (memb) {  // stage the batch: the members are then read by index, not by an unrolled walk of all 16
#pragma unroll
        for (int u = 0; u < kClBatch; ++u) stage[u * NT + tid] = v[u];
      }
      const uint32_t cnt = __popc(memb);
      uint32_t x = cnt;  // inclusive prefix over the lanes
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
      }
      uint32_t base = 0;
      if (lane == 31) base = atomicAdd(&sm.n_list, x);
      base = __shfl_sync(0xffffffffu, base, 31);
      uint32_t pos = base + x - cnt;
      const float* sf = reinterpret_cast<const float*>(stage);
      for (uint32_t m = memb; m != 0u; m &= m - 1u) {  // the raw score bits: keyed after the pass
        const int bit = __ffs(m) - 1, u = bit >> 2, j = bit & 3;
        const float sv = sf[(u * NT + tid) * 4 + j];
        const int o = 32 * (w0 + 4 * u + (lane >> 3)) + 4 * (lane & 7) + j;  // token - c0
        if (pos < (uint32_t)kClListCap) sm.list[pos] = make_uint2(__float_as_uint(sv), (uint32_t)o);
        ++pos;
      }
    };
    constexpr int WB = 4 * kClBatch;  // words per batch
    for (int w0 = wb; w0 < we; w0 += 2 * WB) {
      if (w0 + WB < we) load_batch(vb, w0 + WB);
      process(va, w0);
      if (w0 + WB < we) {
        if (w0 + 2 * WB < we) load_batch(va, w0 + 2 * WB);
        process(vb, w0 + WB);
      }
    }
    __syncthreads();
    // the list's scores as keys, and their digit-2 histogram (from L2 when the list overflowed)
    const uint32_t n1 = sm.n_list;
    if (n1 <= (uint32_t)kClListCap) {
      for (uint32_t i = tid; i < n1; i += kClThreads) {
        const uint32_t key = order_key(__uint_as_float(sm.list[i].x));
        sm.list[i].x = key;
        atomicAdd(&sm.hist[(key >> 10) & (kHistBins - 1)], 1u);
      }
    } else {
      visit_candidates<NT>(srow, c0, c1, rs.lo, rs.hi, [&](int, uint32_t key) {
        if ((key >> 21) == b1) atomicAdd(&sm.hist[(key >> 10) & (kHistBins - 1)], 1u);
      });
    }
    // ---- digit 2: the row's total, from the other CTA's shared histogram in
    // a cluster of two, else through L2 (remote reads of many CTAs' 2048 bins
    // cost more than the atomics and the read-back)
    uint32_t h2[P1];
    if (nc <= 2) {
      cluster.sync();  // every CTA's digit-2 histogram is complete in its shared memory
      const uint32_t* other = nc == 2 ? cluster.map_shared_rank(sm.hist, c ^ 1) : nullptr;
      const int lo = kHistBins - (tid + 1) * P1;  // this thread's bins, ascending
      uint32_t o[P1];
      if constexpr (P1 == 4) {  // one 16-byte read of the other CTA's shared memory
        const uint4 x = other ? *reinterpret_cast<const uint4*>(other + lo) : make_uint4(0u, 0u, 0u, 0u);
        o[0] = x.x; o[1] = x.y; o[2] = x.z; o[3] = x.w;
      } else {
#pragma unroll
        for (int j = 0; j < P1; ++j) o[j] = other ? other[lo + j] : 0u;
      }
#pragma unroll
      for (int j = 0; j < P1; ++j) h2[j] = sm.hist[lo + P1 - 1 - j] + o[P1 - 1 - j];
    } else {
      __syncthreads();
      hist_to_total<NT, kHistBins>(sm.hist, tot);
      cluster.sync();  // the row's digit-2 total is complete in L2
      load_bins_desc<NT, P1>(tot, h2);
    }
    const uint32_t b2 = find_bin_held<NT, P1>(h2, kleft, sm, p.status, above, bcount);
    const uint32_t kleft2 = kleft - above;
    const uint32_t prefix22 = (b1 << 11) | b2;
    const uint32_t n_list = sm.n_list;
    const bool overflow = n_list > (uint32_t)kClListCap;  // the list misses keys: re-read from L2
    if (!overflow) {  // (hist3 was zeroed at the start; the digit-2 search ended with a block barrier)
      for (uint32_t i = tid; i < n_list; i += kClThreads) {
        const uint32_t key = sm.list[i].x;
        if ((key >> 10) == prefix22) atomicAdd(&sm.hist3[key & (kClHist3 - 1)], 1u);
      }
    } else {
      visit_candidates<NT>(srow, c0, c1, rs.lo, rs.hi, [&](int, uint32_t key) {
        if ((key >> 10) == prefix22) atomicAdd(&sm.hist3[key & (kClHist3 - 1)], 1u);
      });
    }
    __syncthreads();
    hist_to_total<NT, kClHist3>(sm.hist3, tot + kHistBins);
    cluster.sync();  // the row's digit-3 total is complete in L2
    // ---- digit 3: the k-th key T and the number of keys equal to T that are kept
    constexpr int P3 = kClHist3 / NT;
    uint32_t h3[P3];
    load_bins_desc<NT, P3>(tot + kHistBins, h3);
    uint32_t ntie_all;
    const uint32_t b3 = find_bin_held<NT, P3>(h3, kleft2, sm, p.status, above, ntie_all);
    const uint32_t T = (prefix22 << 10) | b3;
    const uint32_t quota = kleft2 - above;
    const uint32_t my_ties = sm.hist3[b3];
    uint32_t q_c = my_ties;  // every key equal to T kept (the usual case: one key at T)
    if (ntie_all != quota) {  // the same decision in every CTA of the cluster
      if (tid == 0) slot[c] = my_ties;
      cluster.sync();  // every CTA's count of keys equal to T is posted
      if (tid == 0) {  // ties on the CTAs before this one (lower tokens)
        uint32_t pre = 0;
        for (int j = 0; j < c; ++j) pre += __ldcg(slot + j);
        sm.pre_ties = pre;
      }
      __syncthreads();
      const uint32_t pre = sm.pre_ties;
      q_c = quota > pre ? min(quota - pre, my_ties) : 0u;
    }
    // ---- keys of bin b1 above T into the words; keys equal to T into the words
    // too when this CTA keeps all of its ties (the usual case), else into the
    // tie bitmap
    const bool all_ties = q_c == my_ties;  // uniform in the CTA
    uint32_t* tie_dst = all_ties ? sm.mword : sm.tbits;
    if (!overflow) {
      for (uint32_t i = tid; i < n_list; i += kClThreads) {
        const uint2 e = sm.list[i];
        if (e.x > T)
          atomicOr(&sm.mword[e.y >> 5], 1u << (e.y & 31));
        else if (e.x == T)
          atomicOr(&tie_dst[e.y >> 5], 1u << (e.y & 31));
      }
    } else {
      visit_candidates<NT>(srow, c0, c1, rs.lo, rs.hi, [&](int t, uint32_t key) {
        const int o = t - c0;
        if (key > T && (key >> 21) == b1)
          atomicOr(&sm.mword[o >> 5], 1u << (o & 31));
        else if (key == T)
          atomicOr(&tie_dst[o >> 5], 1u << (o & 31));
      });
    }
    // ---- the first q_c ties of this CTA, in token order
    if (!all_ties && q_c > 0) {  // uniform in the CTA
      __syncthreads();  // the tie bitmap is complete
      constexpr int WPT = kClWordsMax / kClThreads;
      const int w0 = tid * WPT;
      uint32_t cnt = 0;
#pragma unroll
      for (int j = 0; j < WPT; ++j)
        if (w0 + j < nw) cnt += __popc(sm.tbits[w0 + j]);
      uint32_t total;
      uint32_t rank = block_excl_scan<kClThreads>(cnt, total, sm.scan);
#pragma unroll
      for (int j = 0; j < WPT; ++j) {
        if (w0 + j >= nw) break;
        uint32_t x = sm.tbits[w0 + j], keep = 0;
        while (x && rank < q_c) {
          const uint32_t low = x & (~x + 1u);
          keep |= low;
          x ^= low;
          ++rank;
        }
        sm.mword[w0 + j] |= keep;
      }
    }
  } else {
    // ---- no top-k to resolve: sink, window and all or none of the
    // candidates, or the cached top-k of a reusing row (widened by the
    // radius, kept inside the current candidates)
    const int sink_hi = min(p.sink, rs.L), win_lo = max(rs.L - p.window, 0);
    const uint32_t* cm = reused ? p.sc_mask + row * p.mask_words : nullptr;
    const int hi_prev = reused ? p.sc_len[row] - p.window : 0;
    auto cached = [&](int gw) -> uint32_t {
      return (gw < 0 || gw >= p.mask_words) ? 0u : (cm[gw] & range_bits(gw * 32, p.sink, hi_prev));
    };
    for (int w = tid; w < nw; w += kClThreads) {
      const int gw = (c0 >> 5) + w, t0 = gw * 32;
      uint32_t word = range_bits(t0, 0, sink_hi) | range_bits(t0, win_lo, rs.L);
      if (reused) {
        uint32_t x = cached(gw);
        if (p.reuse_radius > 0) {
          const uint32_t prev = cached(gw - 1), next = cached(gw + 1);
          const uint64_t below = ((uint64_t)x << 32) | prev;    // tokens 32(gw-1) .. 32gw+31
          const uint64_t above_w = ((uint64_t)next << 32) | x;  // tokens 32gw .. 32(gw+1)+31
          uint32_t d = x;
          for (int sft = 1; sft <= p.reuse_radius; ++sft)
            d |= (uint32_t)(below >> (32 - sft)) | (uint32_t)(above_w >> sft);
          x = d;
        }
        word |= x & range_bits(t0, rs.lo, rs.hi);
      } else if (rs.mode == 1) {
        word |= range_bits(t0, rs.lo, rs.hi);
      }
      sm.mword[w] = word;
    }
  }

  // ---- write the words once; post kept counts; count check, count, index list
  __syncthreads();
  uint32_t* gm = p.mask + row * p.mask_words + (c0 >> 5);
  const bool refill = p.reuse != nullptr && !reused && rs.mode == 2;  // a fresh top-k refills the cache
  uint32_t kept = 0;
  for (int w = tid; w < nw; w += kClThreads) {
    const uint32_t x = sm.mword[w];
    gm[w] = x;
    if (refill) p.sc_mask[row * p.mask_words + (c0 >> 5) + w] = x;
    kept += __popc(x);
    // every read of this CTA's scores is done: word w's 32 scores are one line
    if (p.discard_scores) discard_l2(srow + c0 + 32 * w);
  }
  // the CTA's kept count, complete in thread 0
  uint32_t kept_cta = __reduce_add_sync(0xffffffffu, kept);
  if (lane == 0) sm.scan[warp] = kept_cta;
  __syncthreads();
  if (warp == 0) kept_cta = __reduce_add_sync(0xffffffffu, lane < kClWarps ? sm.scan[lane] : 0u);
  const int sink_n = min(p.sink, rs.L);
  const uint32_t expect = (uint32_t)(sink_n + (rs.L - max(rs.L - p.window, sink_n)) + rs.k);
  uint32_t* kept_sum = tot + kHistBins + kClHist3;  // 8-byte aligned: kept count (low word), CTA ticket (high)
  if (p.idx == nullptr) {
    // The last CTA of the row to finish (one 64-bit atomic adds this CTA's
    // count and takes its ticket; nothing waits on it) checks the total,
    // writes the count and clears the row's state: every CTA read the
    // histograms and totals before taking its ticket.
    if (tid == 0) {
      __threadfence();
      const unsigned long long old =
          atomicAdd(reinterpret_cast<unsigned long long*>(kept_sum), (1ull << 32) | kept_cta);
      sm.last = (uint32_t)(old >> 32) == (uint32_t)(nc - 1) ? 1u : 0u;
      sm.kept_total = (uint32_t)old + kept_cta;
    }
    __syncthreads();
    if (sm.last) {
      __threadfence();
      if (tid == 0) {
        const uint32_t total = sm.kept_total;
        if (p.count != nullptr) p.count[row] = (int32_t)total;
        // a reused set has the cached top-k's size, not this step's k
        if (!reused && total != expect) atomicOr(p.status, TB_DEV_ERR_COUNT);
      }
      for (int i = tid; i < kHistBins; i += kClThreads) p.hist1[row * kHistBins + i] = 0u;
      for (int i = tid + (nc <= 2 ? kHistBins : 0); i < kClTotWords; i += kClThreads) tot[i] = 0u;  // digit-2 totals unused in pairs
    }
    return;
  }
  // ---- with an index list: the CTAs' kept counts in order give each CTA's offset
  if (tid == 0) slot[kClMaxCluster + c] = kept_cta;
  cluster.sync();  // every CTA's kept count is posted
  uint32_t total = 0, before = 0;
  for (int j = 0; j < nc; ++j) {
    const uint32_t x = __ldcg(slot + kClMaxCluster + j);
    total += x;
    if (j < c) before += x;
  }
  if (c == 0 && tid == 0) {
    if (p.count != nullptr) p.count[row] = (int32_t)total;
    if (!reused && total != expect) atomicOr(p.status, TB_DEV_ERR_COUNT);
  }
  {  // ascending indices: this CTA's run starts after the lower CTAs' kept tokens
    constexpr int WPT = kClWordsMax / kClThreads;
    const int w0 = tid * WPT;
    uint32_t cnt = 0;
#pragma unroll
    for (int j = 0; j < WPT; ++j)
      if (w0 + j < nw) cnt += __popc(sm.mword[w0 + j]);
    uint32_t tot_idx;
    uint32_t pos = before + block_excl_scan<kClThreads>(cnt, tot_idx, sm.scan);
#pragma unroll
    for (int j = 0; j < WPT; ++j) {
      if (w0 + j >= nw) break;
      uint32_t x = sm.mword[w0 + j];
      while (x) {
        const int bit = __ffs(x) - 1;
        x &= x - 1u;
        if (pos < (uint32_t)p.idx_cap) p.idx[row * p.idx_cap + pos] = c0 + 32 * (w0 + j) + bit;
        ++pos;
      }
    }
  }
  if (c == 0) {  // every CTA read the histograms and totals before the last cluster barrier
    for (int i = tid; i < kHistBins; i += kClThreads) p.hist1[row * kHistBins + i] = 0u;
    for (int i = tid + (nc <= 2 ? kHistBins : 0); i < kClTotWords; i += kClThreads) tot[i] = 0u;  // digit-2 totals unused in pairs
  }
}

}  // namespace tb
