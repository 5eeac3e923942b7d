// Sequence-sharded decode: the tokens of each sequence are split into
// contiguous ranges held by ranks in token order (rank r: global tokens
// [t0_r, t0_r + n_r)), and one decode step selects exactly the set that one
// device would (model card "Meta-Llama-3.1-8B-Instruct-Butler", section
// "Method": top-x of the producer's importance scores under a fixed budget,
// plus the sink prefix and the local window; ties to the lower index).
//
// The global k-th largest order key is found with the same three radix
// digits as the one-device selection (11 + 11 + 10 bits), each digit's
// histogram summed over ranks between the passes:
//   shard_hist_kernel   this rank's histogram of the current digit over its
//                       candidates (keys matching the digits found so far);
//   shard_pick_kernel   from the summed histogram, the digit that holds the
//                       k-th key of the row; after the last digit, the
//                       threshold key T and, from every rank's last-digit
//                       count at T (gathered in rank order), this rank's
//                       quota of keys equal to T: ties go to lower indices,
//                       hence to lower ranks first;
//   shard_mask_kernel   this rank's mask words: sink, window, keys above T,
//                       and every key equal to T when the quota is all of them;
//   shard_ties_kernel   rows whose quota is a strict part of their keys
//                       equal to T take the first `quota` of them in index
//                       order (an ordered block scan; rows of ties only).
// Each rank then attends over its part of the set (fp32 partial output and
// log-sum-exp), and merge_partials_kernel combines the gathered partials.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kShardThreads = 256;
constexpr int kShardHistTok = 2048;  // tokens per CTA of the histogram kernel (8 loads per thread)
constexpr int kShardMaskTok = 2048;  // tokens per CTA of the mask kernel (8 warps x 8 words)

struct ShardParams {
  const float* scores;      // [B][rows][max_len] this rank's scores (local token index)
  const uint32_t* hist_in;  // pick: summed histogram [B*rows][2048], or (last digit) [R][B*rows][2048]
  uint32_t* hist;           // hist: [B*rows][2048] this rank's histogram of the current digit
  uint4* state;             // [B*rows]: x key prefix / threshold T, y keys still to take (after the last
                            // digit: this rank's keys equal to T), z mode (0 no top-k, 1 every
                            // candidate, 2 radix), w this rank's quota of keys equal to T
  uint32_t* mask;           // [B][rows][max_len/32]
  uint32_t* status;
  int rows, total_rows, max_len, pass, n_ranks, rank;
  int keep_pct, sink, window;
  int t0;                   // global index of local token 0
  int nloc[kMaxBatch];      // local tokens of sequence b
  int glen[kMaxBatch];      // global length of sequence b
};

// Local candidate range [lo, hi) of sequence b: global candidates
// [sink, L - window) (empty when L - window <= sink) intersected with this
// rank's tokens, in local indices.
__device__ __forceinline__ void shard_cand(const ShardParams& p, int b, int& lo, int& hi) {
  const int L = p.glen[b], n = p.nloc[b];
  const int g_lo = p.sink, g_hi = L - p.window;
  if (g_hi <= g_lo) {
    lo = hi = 0;
    return;
  }
  lo = min(max(g_lo - p.t0, 0), n);
  hi = min(max(g_hi - p.t0, 0), n);
  if (hi < lo) hi = lo;
}

// grid (ceil(max local tokens / kShardHistTok), B*rows); the histogram is
// zeroed before the launch.  Pass 0: the top 11 bits of every candidate's
// order key; pass 1: the next 11 bits of keys whose top 11 bits are the
// row's; pass 2: the low 10 bits of keys whose top 22 bits are the row's.
__global__ void __launch_bounds__(kShardThreads) shard_hist_kernel(const ShardParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint32_t h[kHistBins];
  const int row = blockIdx.y, b = row / p.rows, tid = threadIdx.x;
  int lo, hi;
  shard_cand(p, b, lo, hi);
  const int t_begin = lo + blockIdx.x * kShardHistTok;
  if (t_begin >= hi) return;
  const int t_end = min(hi, t_begin + kShardHistTok);
  uint32_t match = 0;
  int match_shift = 32;
  if (p.pass > 0) {
    const uint4 st = p.state[row];
    if (st.z != 2u) return;
    match_shift = p.pass == 1 ? 21 : 10;
    match = st.x >> match_shift;
  }
  for (int i = tid; i < kHistBins; i += kShardThreads) h[i] = 0;
  __syncthreads();
  const float* s = p.scores + (size_t)row * p.max_len;
  constexpr int PER = kShardHistTok / kShardThreads;
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {  // all loads first, coalesced across the block
    const int t = t_begin + tid + i * kShardThreads;
    v[i] = t < t_end ? s[t] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    if (t_begin + tid + i * kShardThreads >= t_end) break;
    const uint32_t key = order_key(v[i]);
    if (p.pass == 0)
      atomicAdd(&h[key >> 21], 1u);
    else if ((key >> match_shift) == match)
      atomicAdd(&h[p.pass == 1 ? (key >> 10) & 0x7FFu : key & 0x3FFu], 1u);
  }
  __syncthreads();
  for (int i = tid; i < kHistBins; i += kShardThreads)
    if (h[i]) atomicAdd(&p.hist[(size_t)row * kHistBins + i], h[i]);
}

// One CTA per row: the digit of the current pass that holds the row's k-th
// largest key (counts summed over ranks).  Thread t holds the nb/256 bins
// just below nb - t * nb/256 (thread 0 the highest), loaded at once; a
// block scan of the per-thread counts from the top finds the thread, and
// the thread its bin.  Pass 0 also sets the row's mode from the global
// budget k = min(floor(P * L / 100), candidates).  After the last digit the
// threshold T is known, and the gathered per-rank counts of T give this
// rank's quota: the keys equal to T still to take, minus those of lower
// ranks, clamped to this rank's own.  grid B*rows, block 256.
__global__ void __launch_bounds__(kShardThreads) shard_pick_kernel(const ShardParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int NW = kShardThreads / 32;
  __shared__ uint32_t wtot[NW];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int row = blockIdx.x;
  const int b = row / p.rows;
  uint4 st;
  if (p.pass == 0) {
    const int L = p.glen[b];
    const int cand = max(L - p.window - p.sink, 0);
    const int k = (int)min((long long)p.keep_pct * L / 100, (long long)cand);
    st = make_uint4(0u, (uint32_t)k, k == 0 ? 0u : (k == cand ? 1u : 2u), 0u);
    if (st.z != 2u) {
      if (tid == 0) p.state[row] = st;
      return;
    }
  } else {
    st = p.state[row];
    if (st.z != 2u) return;
  }
  const uint32_t krem = st.y;
  const int nb = p.pass == 2 ? 1024 : kHistBins;
  const int per = nb / kShardThreads;  // 8 or 4
  const int nsum = p.pass == 2 ? p.n_ranks : 1;
  const uint32_t* H = p.hist_in + (size_t)row * kHistBins;
  const size_t rstride = (size_t)p.total_rows * kHistBins;
  const int bin_hi = nb - tid * per;  // this thread: bins [bin_hi - per, bin_hi)
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) c[i] = 0;
  for (int r = 0; r < nsum; ++r) {
    const uint32_t* Hr = H + r * rstride + (bin_hi - per);
    if (per == 8) {
      const uint4 a = *reinterpret_cast<const uint4*>(Hr), d = *reinterpret_cast<const uint4*>(Hr + 4);
      c[0] += a.x, c[1] += a.y, c[2] += a.z, c[3] += a.w, c[4] += d.x, c[5] += d.y, c[6] += d.z, c[7] += d.w;
    } else {
      const uint4 a = *reinterpret_cast<const uint4*>(Hr);
      c[0] += a.x, c[1] += a.y, c[2] += a.z, c[3] += a.w;
    }
  }
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) mine += c[i];
  // inclusive scan over threads in order (thread 0 = highest bins)
  uint32_t incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  for (int w = 0; w < warp; ++w) incl += wtot[w];
  uint32_t total = 0;
  for (int w = 0; w < NW; ++w) total += wtot[w];
  const uint32_t excl = incl - mine;
  if (total < krem) {  // the summed counts hold fewer than k keys: inconsistent histograms
    if (tid == 0) {
      atomicOr(p.status, TB_DEV_ERR_COUNT);
      st.z = 0u;
      p.state[row] = st;
    }
    return;
  }
  if (!(excl < krem && krem <= incl)) return;  // exactly one thread goes on
  uint32_t above = excl;
  int i = per - 1;  // c[per - 1] is bin bin_hi - 1, the highest of this thread
  for (; i > 0; --i) {
    if (above + c[i] >= krem) break;
    above += c[i];
  }
  const int bin = bin_hi - per + i;
  const uint32_t rem = krem - above;  // keys of this digit value still to take (>= 1)
  st.x |= (uint32_t)bin << (p.pass == 0 ? 21 : (p.pass == 1 ? 10 : 0));
  if (p.pass < 2) {
    st.y = rem;
  } else {
    uint32_t before = 0;
    for (int r = 0; r < p.rank; ++r) before += H[r * rstride + bin];
    const uint32_t own = H[(size_t)p.rank * rstride + bin];
    st.y = own;
    st.w = rem > before ? min(rem - before, own) : 0u;
  }
  p.state[row] = st;
}

// grid (ceil(max local tokens / kShardMaskTok), B*rows), block 256: each warp
// writes 8 consecutive mask words of its row (one ballot per word; the
// scores of all 8 words are loaded first).  A word
// holds sink tokens, window tokens, every candidate (mode 1), or candidates
// whose key is above T, plus those equal to T when the quota is all of this
// rank's (mode 2).
__global__ void __launch_bounds__(kShardThreads) shard_mask_kernel(const ShardParams p) {
  pdl_wait();
  pdl_trigger();
  const int row = blockIdx.y, b = row / p.rows;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n = p.nloc[b], L = p.glen[b];
  const int nwords = (n + 31) >> 5;
  constexpr int WPW = kShardMaskTok / 32 / (kShardThreads / 32);  // words per warp
  const int w0 = blockIdx.x * (kShardMaskTok / 32) + warp * WPW;
  if (w0 >= nwords) return;
  const uint4 st = p.state[row];
  const int s_end = min(p.sink, L), w_beg = L - p.window;
  const int c_lo = p.sink, c_hi = L - p.window;
  const bool all_eq = st.z == 2u && st.w > 0u && st.w == st.y;
  const float* s = p.scores + (size_t)row * p.max_len;
  uint32_t* m = p.mask + (size_t)row * (p.max_len / 32);
  float v[WPW];
#pragma unroll
  for (int i = 0; i < WPW; ++i) {
    const int tl = (w0 + i) * 32 + lane;
    const int t = p.t0 + tl;
    v[i] = (st.z == 2u && tl < n && t >= c_lo && t < c_hi) ? s[tl] : 0.f;
  }
#pragma unroll
  for (int i = 0; i < WPW; ++i) {
    const int w = w0 + i;
    if (w >= nwords) break;
    const int tl = w * 32 + lane;
    const int t = p.t0 + tl;
    bool keep = false;
    if (tl < n) {
      if (t < s_end || t >= w_beg) {
        keep = true;
      } else if (t >= c_lo && t < c_hi) {
        if (st.z == 1u) {
          keep = true;
        } else if (st.z == 2u) {
          const uint32_t key = order_key(v[i]);
          keep = key > st.x || (all_eq && key == st.x);
        }
      }
    }
    const unsigned bits = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) m[w] = bits;
  }
}

// One CTA per row (grid B*rows, block 256).  Rows whose quota is a strict,
// non-empty part of this rank's keys equal to T take the first `quota` of
// them in index order (block-wide ordered count, 256 tokens per round).
__global__ void __launch_bounds__(kShardThreads) shard_ties_kernel(const ShardParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int NW = kShardThreads / 32;
  __shared__ uint32_t wsum[NW];
  const int row = blockIdx.x, b = row / p.rows;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint4 st = p.state[row];
  if (st.z != 2u || st.w == 0u || st.w >= st.y) return;
  int lo, hi;
  shard_cand(p, b, lo, hi);
  const float* s = p.scores + (size_t)row * p.max_len;
  uint32_t* m = p.mask + (size_t)row * (p.max_len / 32);
  uint32_t taken = 0;  // equal keys met in earlier rounds (the same in every thread)
  for (int base = lo; base < hi && taken < st.w; base += kShardThreads) {
    const int t = base + tid;
    const bool eq = t < hi && order_key(s[t]) == st.x;
    const unsigned bal = __ballot_sync(0xffffffffu, eq);
    if (lane == 0) wsum[warp] = __popc(bal);
    __syncthreads();
    uint32_t before = taken + __popc(bal & ((1u << lane) - 1u)), round = 0;
    for (int w = 0; w < NW; ++w) {
      if (w < warp) before += wsum[w];
      round += wsum[w];
    }
    if (eq && before < st.w) atomicOr(&m[t >> 5], 1u << (t & 31));
    __syncthreads();
    taken += round;
  }
}

// ---------------------------------------------------------------- merge
struct MergeParams {
  const float* parts;  // R blocks of part_stride floats: o [rows][D], then lse [rows] (natural log)
  size_t part_stride;
  void* out;           // [rows][D] kv dtype
  float* lse;          // [rows] or nullptr
  int n_parts, rows;
};

// One warp per (b, h), four per CTA: out = sum_r exp(lse_r - M) o_r /
// sum_r exp(lse_r - M) with M the largest lse_r; parts with lse_r = -inf
// carry no weight; all parts empty: out = 0, lse = -inf.
template <typename T, int D>
__global__ void __launch_bounds__(128) merge_partials_kernel(const MergeParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int DPL = D / 32;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.x * 4 + warp;
  if (row >= p.rows) return;
  const size_t lse_off = (size_t)p.rows * D;
  float M = kNegInf;
  for (int r = 0; r < p.n_parts; ++r) M = fmaxf(M, p.parts[r * p.part_stride + lse_off + row]);
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  float wsum = 0.f;
  if (M != kNegInf) {
    for (int r = 0; r < p.n_parts; ++r) {
      const float* part = p.parts + r * p.part_stride;
      const float l = part[lse_off + row];
      if (l == kNegInf) continue;
      const float w = expf(l - M);
      wsum += w;
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[i] = fmaf(w, part[(size_t)row * D + lane + 32 * i], acc[i]);
    }
  }
  const float inv = M == kNegInf ? 0.f : 1.f / wsum;
#pragma unroll
  for (int i = 0; i < DPL; ++i) reinterpret_cast<T*>(p.out)[(size_t)row * D + lane + 32 * i] = from_f32<T>(acc[i] * inv);
  if (p.lse != nullptr && lane == 0) p.lse[row] = M == kNegInf ? kNegInf : M + logf(wsum);
}

}  // namespace tb
