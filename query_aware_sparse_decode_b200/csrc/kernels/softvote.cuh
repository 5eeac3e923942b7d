// Soft-voting variant of the selection (TokenSelect README, "Dynamic
// Token-Level KV Cache Selection" and "Per-head Soft Voting Mechanism"):
//
//   a[h][t] = q[b][h] . K[b][g(h)][t] / sqrt(D),   t < len[b]
//   p[h][t] = softmax_t(a[h][.]),   votes[b][t] = sum_h p[h][t]
//
// One shared ranking per sequence; the selection then reuses the top-k
// kernel on `votes` (one row per sequence) and the sparse attention kernel in
// shared-mask mode.
//
// softvote_logits: HBM stream over K (each row read once per KV head and
// shared by the group's query heads), contiguous 16-token tiles gathered by
// cp.async into a swizzled ring, q . K^T on mma.sync (bf16 in, fp32
// accumulate); writes the logits in the log2 domain and one (max, sum of
// 2^(a - max)) pair per head and chunk.  The last CTA of a sequence to finish
// (a device-scope completion counter, fence then count; nothing waits on it)
// merges the sequence's chunk pairs into each head's (M, 1/Z) and resets the
// counter for the next launch.
// softvote_reduce: sums 2^(a - M) / Z over the heads, one token per thread
// (logits are L2-resident), after one read of the heads' (M, 1/Z).  Optionally it also
// builds the first-digit histogram of the votes over the candidate range
// [sink, len - window) for the selection that follows (warp-aggregated shared
// atomics: votes crowd into few bins).
#pragma once

#include "attn.cuh"
#include "common.cuh"

namespace tb {

// Tokens per CTA of the logits pass: chosen per launch (a multiple of 16, at
// least kVoteMinChunk) so that the grid is about four CTAs per SM in one wave.
constexpr int kVoteMinChunk = 256;

struct VoteParams {
  const void* k_cache;  // [B][Hkv][max_len][D] bf16, or a page pool (KvLayout)
  KvLayout kl;
  const void* q;        // [B][Hq][D] bf16
  float* logits;        // [B][Hq][max_len], log2 domain
  float* stats;         // [B][Hq][nchunk][2]
  float* mz;            // [B][Hq][2]: each head's merged max M (log2 domain) and 1/Z
  uint32_t* done;       // [B] logits CTAs finished (zero between launches)
  float* votes;         // [B][max_len]
  uint32_t* hist1;      // [B][2048] first-digit histograms of the votes, or nullptr
  int Hq, Hkv, max_len, nchunk;  // nchunk: stride of the chunk statistics, >= max_len / chunk
  int chunk;                     // tokens per CTA of the logits pass
  int sink, window;
  float scale_log2;
  int lens[kMaxBatch];
};

template <int D, int GS>
__global__ void __launch_bounds__(kAttnThreads, 2) softvote_logits_kernel(const VoteParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int ROWB = D * 2;
  constexpr int NCH = D / 8;
  constexpr int STAGE = kAttnTile * ROWB;  // K only
  constexpr int KSTEPS = D / 16;
  extern __shared__ __align__(128) uint8_t smem[];
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = p.lens[b];
  const int t0 = chunk * p.chunk;
  if (t0 >= L) return;
  const int t1 = min(t0 + p.chunk, L);
  const int n = t1 - t0;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 2, tq = lane & 3;
  const uint8_t* Kb = reinterpret_cast<const uint8_t*>(p.k_cache);  // rows via kv_row

  uint32_t qa[KSTEPS][2];
  {
    const __nv_bfloat16* qrow =
        reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + g * GS + (grp < GS ? grp : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      const int dim = (4 * (kk / 2) + tq) * 8 + (kk % 2) * 4;
      qa[kk][0] = grp < GS ? *reinterpret_cast<const uint32_t*>(qrow + dim) : 0u;
      qa[kk][1] = grp < GS ? *reinterpret_cast<const uint32_t*>(qrow + dim + 2) : 0u;
    }
  }
  float m_run = kNegInf, l_run = 0.f;
  const int ntiles = (n + kAttnTile - 1) / kAttnTile;
  const int my_n = ntiles > warp ? (ntiles - warp + kAttnWarps - 1) / kAttnWarps : 0;
  uint8_t* my_ring = smem + warp * kAttnStages * STAGE;
  // A tile's 16 tokens are consecutive cache rows: tiles start at multiples of
  // 16 and pages hold a power of two >= 16 tokens, so one row lookup per tile
  // serves all of them (rows past the ragged end repeat the last token).
  auto issue = [&](int it) {
    const int tile = warp + it * kAttnWarps;
    uint8_t* sb = my_ring + (it % kAttnStages) * STAGE;
    const int tt = t0 + tile * kAttnTile;
    const int last = t1 - 1 - tt;
    const uint8_t* base = Kb + (size_t)kv_row(p.kl, b, g, p.Hkv, p.max_len, tt) * ROWB;
#pragma unroll
    for (int c = lane; c < kAttnTile * NCH; c += 32) {
      const int row = c / NCH, part = c % NCH;
      cp_async_16(sb + row * ROWB + ((part ^ (row & 7)) << 4), base + min(row, last) * ROWB + part * 16);
    }
  };
#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) {
    if (s < my_n) issue(s);
    cp_async_commit();
  }
  const size_t lrow = ((size_t)b * p.Hq + g * GS + (grp < GS ? grp : 0)) * p.max_len;
  for (int it = 0; it < my_n; ++it) {
    if (it + kAttnStages - 1 < my_n) issue(it + kAttnStages - 1);
    cp_async_commit();
    cp_async_wait<kAttnStages - 1>();
    __syncwarp();
    const uint8_t* Ks = my_ring + (it % kAttnStages) * STAGE;
    const int tile = warp + it * kAttnWarps;
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int c = 4 * i + tq;
      const uint4 k0 = *reinterpret_cast<const uint4*>(Ks + grp * ROWB + ((c ^ (grp & 7)) << 4));
      const uint4 k1 = *reinterpret_cast<const uint4*>(Ks + (grp + 8) * ROWB + ((c ^ (grp & 7)) << 4));
      mma_16816(acc0, qa[2 * i][0], 0u, qa[2 * i][1], 0u, k0.x, k0.y);
      mma_16816(acc0, qa[2 * i + 1][0], 0u, qa[2 * i + 1][1], 0u, k0.z, k0.w);
      mma_16816(acc1, qa[2 * i][0], 0u, qa[2 * i][1], 0u, k1.x, k1.y);
      mma_16816(acc1, qa[2 * i + 1][0], 0u, qa[2 * i + 1][1], 0u, k1.z, k1.w);
    }
    const int tb0 = t0 + tile * kAttnTile;
    const int ta = tb0 + 2 * tq, tc = tb0 + 2 * tq + 8;
    const bool real = grp < GS;
    const float s0 = real && ta < t1 ? acc0[0] * p.scale_log2 : kNegInf;
    const float s1 = real && ta + 1 < t1 ? acc0[1] * p.scale_log2 : kNegInf;
    const float s2 = real && tc < t1 ? acc1[0] * p.scale_log2 : kNegInf;
    const float s3 = real && tc + 1 < t1 ? acc1[1] * p.scale_log2 : kNegInf;
    if (real) {
      if (ta + 1 < t1) {
        *reinterpret_cast<float2*>(p.logits + lrow + ta) = make_float2(s0, s1);
      } else if (ta < t1) {
        p.logits[lrow + ta] = s0;
      }
      if (tc + 1 < t1) {
        *reinterpret_cast<float2*>(p.logits + lrow + tc) = make_float2(s2, s3);
      } else if (tc < t1) {
        p.logits[lrow + tc] = s2;
      }
    }
    float mt = fmaxf(fmaxf(s0, s1), fmaxf(s2, s3));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const float m_new = fmaxf(m_run, mt);
    if (m_new != kNegInf) {
      // 2^x on the special-function unit (relative error about 2^-22, far
      // inside the votes' tolerance); 2^-inf = 0
      l_run = l_run * fast_exp2(m_run - m_new) + fast_exp2(s0 - m_new) + fast_exp2(s1 - m_new) +
              fast_exp2(s2 - m_new) + fast_exp2(s3 - m_new);
      m_run = m_new;
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();
  float* wm = reinterpret_cast<float*>(smem);
  float* wl = wm + kAttnWarps * GS;
  if (grp < GS && tq == 0) {
    wm[warp * GS + grp] = m_run;
    wl[warp * GS + grp] = l_run;
  }
  __syncthreads();
  if (tid < GS) {
    float M = kNegInf;
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, wm[w * GS + tid]);
    float l = 0.f;
    if (M != kNegInf)
      for (int w = 0; w < kAttnWarps; ++w)
        if (wm[w * GS + tid] != kNegInf) l += wl[w * GS + tid] * exp2f(wm[w * GS + tid] - M);
    const size_t ph = (((size_t)b * p.Hq + g * GS + tid) * p.nchunk + chunk) * 2;
    p.stats[ph] = M;
    p.stats[ph + 1] = l;
  }
  // ---- the sequence's last CTA merges every chunk's pair into (M, 1/Z) per head
  __shared__ uint32_t s_last;
  __threadfence();  // this CTA's pairs are visible device-wide before it is counted
  __syncthreads();
  const int nch = (L + p.chunk - 1) / p.chunk;
  if (tid == 0) s_last = atomicAdd(&p.done[b], 1u) == (uint32_t)(nch * p.Hkv - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // four threads per head (consecutive lanes), each merging every fourth chunk
  constexpr int TPH = 4;
  const int sub = tid % TPH;
  for (int h0 = 0; h0 < p.Hq; h0 += kAttnThreads / TPH) {
    const int h = h0 + tid / TPH;
    float m = kNegInf, l = 0.f;
    if (h < p.Hq) {
      const float2* st = reinterpret_cast<const float2*>(p.stats + ((size_t)b * p.Hq + h) * p.nchunk * 2);
#pragma unroll 4
      for (int c = sub; c < nch; c += TPH) {
        const float2 e = __ldcg(st + c);
        if (e.x == kNegInf) continue;
        const float mn = fmaxf(m, e.x);
        l = l * exp2f(m - mn) + e.y * exp2f(e.x - mn);
        m = mn;
      }
    }
#pragma unroll
    for (int o = 1; o < TPH; o <<= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o), l2 = __shfl_xor_sync(0xffffffffu, l, o);
      const float mn = fmaxf(m, m2);
      if (mn != kNegInf) {
        l = (m == kNegInf ? 0.f : l * exp2f(m - mn)) + (m2 == kNegInf ? 0.f : l2 * exp2f(m2 - mn));
        m = mn;
      }
    }
    if (h < p.Hq && sub == 0) {
      p.mz[((size_t)b * p.Hq + h) * 2] = m;
      p.mz[((size_t)b * p.Hq + h) * 2 + 1] = 1.f / l;
    }
  }
  if (tid == 0) p.done[b] = 0u;  // ready for the next launch (stream-ordered after this grid)
}

// grid (ceil(max len / 256), B), block 256: one token per thread.  The
// token's logits of the first kVotePrefetch heads are requested before the
// CTA reads the heads' (M, 1/Z), so the two latencies overlap.
constexpr int kVoteMaxHeads = 128;
constexpr int kVoteReduceTok = 256;
constexpr int kVotePrefetch = 32;
__global__ void __launch_bounds__(256) softvote_reduce_kernel(const VoteParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float2 sMZ[kVoteMaxHeads];  // per head: (M, 1/Z)
  __shared__ uint32_t hist[kHistBins];
  const int b = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int L = p.lens[b];
  const int t_begin = blockIdx.x * kVoteReduceTok;
  if (t_begin >= L) return;
  const int t = t_begin + tid;
  const float* lg = p.logits + (size_t)b * p.Hq * p.max_len + t;
  float a[kVotePrefetch];
#pragma unroll
  for (int h = 0; h < kVotePrefetch; ++h) a[h] = (h < p.Hq && t < L) ? lg[(size_t)h * p.max_len] : 0.f;
  for (int h = tid; h < p.Hq; h += 256) {
    const float2 mz = reinterpret_cast<const float2*>(p.mz)[(size_t)b * p.Hq + h];
    sMZ[h] = mz;
  }
  if (p.hist1 != nullptr)
    for (int i = tid; i < kHistBins; i += 256) hist[i] = 0;
  __syncthreads();
  float v = 0.f;  // sum over the heads in head order
  if (t < L) {
#pragma unroll
    for (int h = 0; h < kVotePrefetch; ++h)
      if (h < p.Hq) {
        const float2 mz = sMZ[h];
        v = fmaf(fast_exp2(a[h] - mz.x), mz.y, v);
      }
    for (int h = kVotePrefetch; h < p.Hq; ++h) {
      const float2 mz = sMZ[h];
      v = fmaf(fast_exp2(lg[(size_t)h * p.max_len] - mz.x), mz.y, v);
    }
    p.votes[(size_t)b * p.max_len + t] = v;
  }
  if (p.hist1 == nullptr) return;
  const bool in = t < L && t >= p.sink && t < L - p.window;
  const uint32_t bin = in ? (order_key(v) >> 21) : 0xFFFFFFFFu;
  const uint32_t peers = __match_any_sync(0xffffffffu, bin);
  if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
  __syncthreads();
  for (int i = tid; i < kHistBins; i += 256)
    if (hist[i]) atomicAdd(&p.hist1[(size_t)b * kHistBins + i], hist[i]);
}

}  // namespace tb
