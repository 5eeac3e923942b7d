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
// cp.async into a swizzled ring, K q^T on mma.sync (bf16 in, fp32
// accumulate; the tile's tokens as the M rows, the group's heads as the N
// columns); writes the logits in the log2 domain and one (max, sum of
// 2^(a - max)) pair per head and chunk.
// softvote_reduce: merges each head's chunk pairs into (M, 1/Z) (every CTA,
// while its first logits are in flight), then sums 2^(a - M) / Z over the
// heads, one token per thread (logits are L2-resident), and drops the
// CTA's logit lines from L2 unwritten (no reader follows).  Optionally it also
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
constexpr int kVoteWarps = 4;   // warps per CTA of the logits pass
constexpr int kVoteThreads = kVoteWarps * 32;
constexpr int kVoteStages = 3;  // ring stages per warp of the logits pass (16 K rows each)
template <int D>
constexpr int vote_logits_smem() { return kVoteWarps * kVoteStages * kAttnTile * D * 2; }

struct VoteParams {
  const void* k_cache;  // [B][Hkv][max_len][D] bf16, or a page pool (KvLayout)
  KvLayout kl;
  const void* q;        // [B][Hq][D] bf16
  float* logits;        // [B][Hq][max_len], log2 domain
  float* stats;         // [B][Hq][nchunk][2]
  float* votes;         // [B][max_len]
  uint32_t* hist1;      // [B][2048] first-digit histograms of the votes, or nullptr
  int Hq, Hkv, max_len, nchunk;  // nchunk: stride of the chunk statistics, >= max_len / chunk
  int chunk;                     // tokens per CTA of the logits pass
  int sink, window;
  float scale_log2;
  int lens[kMaxBatch];
};

template <int D, int GS>
__global__ void __launch_bounds__(kVoteThreads, 2) softvote_logits_kernel(const VoteParams p) {
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

  // S^T = K Q^T on mma.sync: the tile's 16 tokens are the M rows (A = the K
  // tile, ldmatrix), the group's heads the 8 N columns (B = Q^T, heads >= GS
  // zero).  Lane (grp, tq) holds head grp, dims 16kk + 2tq + {0,1} and
  // 16kk + 8 + 2tq + {0,1} of Q^T, and receives the logits of tokens grp and
  // grp + 8 for heads 2tq and 2tq + 1.
  uint32_t qb[KSTEPS][2];
  {
    const __nv_bfloat16* qrow =
        reinterpret_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + g * GS + (grp < GS ? grp : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      qb[kk][0] = grp < GS ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * tq) : 0u;
      qb[kk][1] = grp < GS ? *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 8 + 2 * tq) : 0u;
    }
  }
  // the lane's two heads, and whether each is one of the group's
  const int hp = 2 * tq;
  const bool real0 = hp < GS, real1 = hp + 1 < GS;
  // per lane and head: running max and sum of 2^(a - max) over the lane's tokens
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};
  const int ntiles = (n + kAttnTile - 1) / kAttnTile;
  const int my_n = ntiles > warp ? (ntiles - warp + kVoteWarps - 1) / kVoteWarps : 0;
  uint8_t* my_ring = smem + warp * kVoteStages * STAGE;
  const uint32_t ring_u32 = smem_u32(my_ring);
  // ldmatrix rows: lane supplies row (lane & 7) of matrix (lane >> 3) = tokens
  // 8 (j & 1) + r, piece 2kk + (j >> 1); the swizzled piece is 2kk ^ ((j >> 1) ^ r)
  const int lr = lane & 7, lj = lane >> 3;
  const uint32_t k_row_off = (uint32_t)((lr + 8 * (lj & 1)) * ROWB);
  const uint32_t k_x = (uint32_t)(((lj >> 1) ^ lr) << 4);
  // A tile's 16 tokens are consecutive cache rows: tiles start at multiples of
  // 16 and pages hold a power of two >= 16 tokens, so one row lookup per tile
  // serves all of them (rows past the ragged end repeat the last token).
  auto issue = [&](int it) {
    const int tile = warp + it * kVoteWarps;
    uint8_t* sb = my_ring + (it % kVoteStages) * STAGE;
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
  for (int s = 0; s < kVoteStages - 1; ++s) {
    if (s < my_n) issue(s);
    cp_async_commit();
  }
  float* lrow0 = p.logits + ((size_t)b * p.Hq + g * GS + (real0 ? hp : 0)) * p.max_len;
  float* lrow1 = p.logits + ((size_t)b * p.Hq + g * GS + (real1 ? hp + 1 : 0)) * p.max_len;
  for (int it = 0; it < my_n; ++it) {
    if (it + kVoteStages - 1 < my_n) issue(it + kVoteStages - 1);
    cp_async_commit();
    cp_async_wait<kVoteStages - 1>();
    __syncwarp();
    const uint32_t st = ring_u32 + (uint32_t)((it % kVoteStages) * STAGE);
    const int tile = warp + it * kVoteWarps;
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t a[4];
      ldsm_x4(a, st + k_row_off + (((uint32_t)(32 * kk)) ^ k_x));
      mma_16816(s, a[0], a[1], a[2], a[3], qb[kk][0], qb[kk][1]);
    }
    __syncwarp();  // the stage is refilled by the next iteration's copies
    const int ta = t0 + tile * kAttnTile + grp, tc = ta + 8;
    // x[0], x[1]: token ta, heads hp, hp + 1; x[2], x[3]: token tc
    float x[4];
    x[0] = ta < t1 ? s[0] * p.scale_log2 : kNegInf;
    x[1] = ta < t1 ? s[1] * p.scale_log2 : kNegInf;
    x[2] = tc < t1 ? s[2] * p.scale_log2 : kNegInf;
    x[3] = tc < t1 ? s[3] * p.scale_log2 : kNegInf;
    if (real0) {
      if (ta < t1) lrow0[ta] = x[0];
      if (tc < t1) lrow0[tc] = x[2];
    }
    if (real1) {
      if (ta < t1) lrow1[ta] = x[1];
      if (tc < t1) lrow1[tc] = x[3];
    }
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float mn = fmaxf(m_run[e], fmaxf(x[e], x[2 + e]));
      if (mn != kNegInf) {
        // 2^x on the special-function unit (relative error about 2^-22, far
        // inside the votes' tolerance); 2^-inf = 0
        l_run[e] = l_run[e] * fast_exp2(m_run[e] - mn) + fast_exp2(x[e] - mn) + fast_exp2(x[2 + e] - mn);
        m_run[e] = mn;
      }
    }
  }
  cp_async_wait<0>();
  // merge the lanes' pairs of each head (the 8 lanes with the same tq)
#pragma unroll
  for (int e = 0; e < 2; ++e)
#pragma unroll
    for (int o = 4; o < 32; o <<= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m_run[e], o), l2 = __shfl_xor_sync(0xffffffffu, l_run[e], o);
      const float mn = fmaxf(m_run[e], m2);
      if (mn != kNegInf) {
        l_run[e] = (m_run[e] == kNegInf ? 0.f : l_run[e] * exp2f(m_run[e] - mn)) +
                   (m2 == kNegInf ? 0.f : l2 * exp2f(m2 - mn));
        m_run[e] = mn;
      }
    }
  __syncthreads();
  float* wm = reinterpret_cast<float*>(smem);
  float* wl = wm + kVoteWarps * GS;
  if (grp == 0) {
    if (real0) {
      wm[warp * GS + hp] = m_run[0];
      wl[warp * GS + hp] = l_run[0];
    }
    if (real1) {
      wm[warp * GS + hp + 1] = m_run[1];
      wl[warp * GS + hp + 1] = l_run[1];
    }
  }
  __syncthreads();
  if (tid < GS) {
    float M = kNegInf;
    for (int w = 0; w < kVoteWarps; ++w) M = fmaxf(M, wm[w * GS + tid]);
    float l = 0.f;
    if (M != kNegInf)
      for (int w = 0; w < kVoteWarps; ++w)
        if (wm[w * GS + tid] != kNegInf) l += wl[w * GS + tid] * exp2f(wm[w * GS + tid] - M);
    const size_t ph = (((size_t)b * p.Hq + g * GS + tid) * p.nchunk + chunk) * 2;
    p.stats[ph] = M;
    p.stats[ph + 1] = l;
  }
}

// grid (ceil(max len / 256), B), block 256: one token per thread.  The
// token's logits of the first kVotePrefetch heads are requested before the
// CTA merges the heads' chunk pairs, so the two latencies overlap.
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
  // each head's (M, 1/Z) from the logits pass's per-chunk pairs: eight
  // threads per head, each merging every eighth chunk, then across the eight
  const int nch = (L + p.chunk - 1) / p.chunk;
  constexpr int TPH = 8;
  for (int h0 = 0; h0 < p.Hq; h0 += 256 / TPH) {
    const int h = h0 + tid / TPH, sub = tid % TPH;
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
    if (h < p.Hq && sub == 0) sMZ[h] = make_float2(m, 1.f / l);
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
  // The logits are a dead intermediate once every thread has read its own:
  // the CTA's lines (256 tokens = eight 128-byte lines per head) are dropped
  // from L2 without a write-back.
  __syncthreads();
  for (int e = tid; e < p.Hq * (kVoteReduceTok / 32); e += 256)
    discard_l2(p.logits + ((size_t)b * p.Hq + e / (kVoteReduceTok / 32)) * p.max_len + t_begin +
               32 * (e % (kVoteReduceTok / 32)));
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
