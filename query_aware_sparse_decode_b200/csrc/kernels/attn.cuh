// butler_sparse_attn + butler_attn_combine: exact attention over a selected
// token set of the untouched full KV cache (model card
// "Meta-Llama-3.1-8B-Instruct-Butler": sparse attention with a fixed budget
// while preserving the full KV cache; TokenButler abstract, same statement).
//
//   o[b][h] = sum_{t in Sel[b][h]} softmax_t(q[b][h] . K[b][g][t] / sqrt(D)) V[b][g][t]
//
// Split-K flash decoding: a CTA owns (b, KV head g, chunk of tokens).  It
// ORs the selection masks of the group's Hq/Hkv query heads, so every K/V
// row of the group's union is gathered from HBM exactly once and serves all
// heads (a per-token head bitmask masks the scores).  Rows are gathered by
// cp.async into an XOR-swizzled shared-memory ring (3 stages per warp).
// QK^T and PV run on mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the
// group's heads as the M rows; the online softmax is kept in fp32 in the
// log2 domain.  Each CTA writes one (m, l, o) partial per head; the combine
// kernel merges the chunks with an fp32 log-sum-exp.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kAttnWarps = 4;
constexpr int kAttnThreads = kAttnWarps * 32;
constexpr int kAttnStages = 3;
constexpr int kAttnTile = 16;        // tokens per mma tile
constexpr int kAttnMaxChunk = 2048;  // tokens per gather list (a CTA's chunk may span several)

struct AttnParams {
  const void* k_cache;   // [B][Hkv][max_len][D], or a page pool (KvLayout)
  const void* v_cache;
  KvLayout kl;
  const void* q;         // [B][Hq][D]
  const uint32_t* mask;  // per mask_mode
  float* part_o;         // [B][Hq][nsplit][D]
  float* part_ml;        // [B][Hq][nsplit][2]: running max (log2 domain), sum
  uint32_t* status;
  int mask_mode, mask_words;
  int Hq, Hkv, max_len, chunk, nsplit;
  float scale_log2;      // log2(e) / sqrt(D)
  int lens[kMaxBatch];
};

// Builds the CTA's gather list: the cache rows of the ascending union tokens
// of [t0, t1) with a head bitmask each; pads to a multiple of 16 with
// (row of t0, no head).
template <int GS>
__device__ __forceinline__ int build_union_list(const AttnParams& p, int b, int g, int t0, int t1, int32_t* list_idx,
                                                uint8_t* list_hb, uint32_t* scan_sm) {
  const int tid = threadIdx.x;
  const int nwords = (t1 - t0 + 31) >> 5;
  const int w_base = t0 >> 5;
  int base = 0;
  for (int w0 = 0; w0 < nwords; w0 += kAttnThreads) {
    const int w = w0 + tid;
    uint32_t u = 0;
    uint32_t hm[GS];
#pragma unroll
    for (int hh = 0; hh < GS; ++hh) hm[hh] = 0;
    if (w < nwords) {
      if (p.mask_mode == TB_MASK_PER_HEAD) {
#pragma unroll
        for (int hh = 0; hh < GS; ++hh) {
          hm[hh] = p.mask[((size_t)b * p.Hq + g * GS + hh) * p.mask_words + w_base + w];
          u |= hm[hh];
        }
      } else if (p.mask_mode == TB_MASK_SHARED) {
        u = p.mask[(size_t)b * p.mask_words + w_base + w];
      } else if (p.mask_mode == TB_MASK_GROUP) {
        u = p.mask[((size_t)b * p.Hkv + g) * p.mask_words + w_base + w];
      } else {
        u = 0xFFFFFFFFu;
      }
      const int valid = t1 - (t0 + 32 * w);
      if (valid < 32) u &= (1u << valid) - 1u;
    }
    uint32_t total;
    int pos = base + (int)block_excl_scan<kAttnThreads>(__popc(u), total, scan_sm);
    while (u) {
      const int j = __ffs(u) - 1;
      u &= u - 1u;
      uint32_t hb = 0xFFu;
      if (p.mask_mode == TB_MASK_PER_HEAD) {
        hb = 0;
#pragma unroll
        for (int hh = 0; hh < GS; ++hh) hb |= ((hm[hh] >> j) & 1u) << hh;
      }
      list_idx[pos] = (int32_t)kv_row(p.kl, b, g, p.Hkv, p.max_len, t0 + 32 * w + j);  // the token's cache row
      list_hb[pos] = (uint8_t)hb;
      ++pos;
    }
    base += (int)total;
  }
  const int padded = (base + kAttnTile - 1) / kAttnTile * kAttnTile;
  for (int i = base + tid; i < padded; i += kAttnThreads) {
    list_idx[i] = (int32_t)kv_row(p.kl, b, g, p.Hkv, p.max_len, t0);
    list_hb[i] = 0;
  }
  __syncthreads();
  return base;
}

// Writes the CTA's merged (m, l, o) partial for each head of the group from
// per-warp states held in shared memory.
template <int D, int GS>
__device__ __forceinline__ void write_partial(const AttnParams& p, int b, int g, int split, const float* wm,
                                              const float* wl, const float* wo) {
  for (int e = threadIdx.x; e < GS * D; e += kAttnThreads) {
    const int hh = e / D, d = e % D;
    float M = kNegInf;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, wm[w * GS + hh]);
    float o = 0.f, l = 0.f;
    if (M != kNegInf) {
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float m = wm[w * GS + hh];
        const float f = m == kNegInf ? 0.f : exp2f(m - M);
        o += f * wo[(w * GS + hh) * D + d];
        l += f * wl[w * GS + hh];
      }
    }
    const size_t ph = ((size_t)b * p.Hq + g * GS + hh) * p.nsplit + split;
    p.part_o[ph * D + d] = o;
    if (d == 0) {
      p.part_ml[ph * 2] = M;
      p.part_ml[ph * 2 + 1] = l;
    }
  }
}


constexpr int kMaxSplits = 512;

// ---------------------------------------------------------------- bf16 / mma.sync
template <int D>
constexpr int attn_bf16_smem_bytes() {
  return kAttnWarps * kAttnStages * 2 * kAttnTile * D * 2 + (kAttnMaxChunk + kAttnTile) * 5;
}

template <int D, int GS>
__global__ void __launch_bounds__(kAttnThreads, 2) attn_bf16_kernel(const AttnParams p) {
  pdl_wait();
  pdl_trigger();
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(GS >= 1 && GS <= 8, "group size");
  constexpr int ROWB = D * 2;                       // bytes per K or V row
  constexpr int NCH = D / 8;                        // 16-byte pieces per row
  constexpr int STAGE = 2 * kAttnTile * ROWB;       // K tile + V tile
  constexpr int KSTEPS = D / 16;
  constexpr int NT = D / 8;                         // n-tiles of the output
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* ring = smem;
  int32_t* list_idx = reinterpret_cast<int32_t*>(smem + kAttnWarps * kAttnStages * STAGE);
  uint8_t* list_hb = reinterpret_cast<uint8_t*>(list_idx + kAttnMaxChunk + kAttnTile);
  __shared__ uint32_t scan_sm[32];

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = p.lens[b];
  const int t0 = split * p.chunk;
  if (t0 >= L) return;
  const int t1 = min(t0 + p.chunk, L);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = lane >> 2, tq = lane & 3;
  // gather lists hold cache rows (dense or paged), so the bases are the caches'
  const uint8_t* Kb = reinterpret_cast<const uint8_t*>(p.k_cache);
  const uint8_t* Vb = reinterpret_cast<const uint8_t*>(p.v_cache);

  // A fragments of Q (rows = the group's heads; rows >= GS and 8..15 are 0).
  // Logical k (2tq + {0,1}) of k-step kk maps to dims (4(kk/2)+tq)*8 + (kk%2)*4 + {0,1},
  // logical k (2tq + 8 + {0,1}) to the same + {2,3}; K uses the same map.
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

  float o[NT][2];
#pragma unroll
  for (int j = 0; j < NT; ++j) o[j][0] = o[j][1] = 0.f;
  float m_run = kNegInf, l_run = 0.f;
  uint8_t* my_ring = ring + warp * kAttnStages * STAGE;

  // the CTA's chunk is processed in sub-chunks of up to kAttnMaxChunk tokens
  // (one gather list each); the softmax state carries across them
  for (int sc0 = t0; sc0 < t1; sc0 += kAttnMaxChunk) {
  const int n = build_union_list<GS>(p, b, g, sc0, min(sc0 + kAttnMaxChunk, t1), list_idx, list_hb, scan_sm);
  const int ntiles = n / kAttnTile + (n % kAttnTile ? 1 : 0);
  const int my_n = ntiles > warp ? (ntiles - warp + kAttnWarps - 1) / kAttnWarps : 0;

  // A lane copies the same 16-byte pieces of its rows from K and from V: the
  // rows' cache indices are read from the list once, before the copies.
  constexpr int PER = kAttnTile * NCH / 32;  // pieces per lane and tensor
  auto issue = [&](int it) {
    const int tile = warp + it * kAttnWarps;
    uint8_t* sb = my_ring + (it % kAttnStages) * STAGE;
    int tok[PER];
#pragma unroll
    for (int i = 0; i < PER; ++i) tok[i] = list_idx[tile * kAttnTile + (lane + 32 * i) / NCH];
#pragma unroll
    for (int tensor = 0; tensor < 2; ++tensor) {
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const int rc = lane + 32 * i, row = rc / NCH, part = rc % NCH;
        cp_async_16(sb + tensor * kAttnTile * ROWB + row * ROWB + ((part ^ (row & 7)) << 4),
                    (tensor ? Vb : Kb) + (size_t)tok[i] * ROWB + part * 16);
      }
    }
  };
#pragma unroll
  for (int s = 0; s < kAttnStages - 1; ++s) {
    if (s < my_n) issue(s);
    cp_async_commit();
  }

  for (int it = 0; it < my_n; ++it) {
    if (it + kAttnStages - 1 < my_n) issue(it + kAttnStages - 1);
    cp_async_commit();
    cp_async_wait<kAttnStages - 1>();
    __syncwarp();
    const uint8_t* Ks = my_ring + (it % kAttnStages) * STAGE;
    const uint8_t* Vs = Ks + kAttnTile * ROWB;
    const int tile = warp + it * kAttnWarps;

    // ---- S = Q K^T for tokens 0..7 (acc0) and 8..15 (acc1) of the tile
    float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int i = 0; i < D / 32; ++i) {
      const int c = 4 * i + tq;
      const uint4 k0 = *reinterpret_cast<const uint4*>(Ks + grp * ROWB + ((c ^ (grp & 7)) << 4));
      const uint4 k1 = *reinterpret_cast<const uint4*>(Ks + (grp + 8) * ROWB + ((c ^ ((grp + 8) & 7)) << 4));
      mma_16816(acc0, qa[2 * i][0], 0u, qa[2 * i][1], 0u, k0.x, k0.y);
      mma_16816(acc0, qa[2 * i + 1][0], 0u, qa[2 * i + 1][1], 0u, k0.z, k0.w);
      mma_16816(acc1, qa[2 * i][0], 0u, qa[2 * i][1], 0u, k1.x, k1.y);
      mma_16816(acc1, qa[2 * i + 1][0], 0u, qa[2 * i + 1][1], 0u, k1.z, k1.w);
    }

    // ---- masked online softmax (log2 domain) for head row `grp`
    const uint8_t* hb = list_hb + tile * kAttnTile;
    const bool real = grp < GS;
    const float s0 = real && ((hb[2 * tq] >> grp) & 1) ? acc0[0] * p.scale_log2 : kNegInf;
    const float s1 = real && ((hb[2 * tq + 1] >> grp) & 1) ? acc0[1] * p.scale_log2 : kNegInf;
    const float s2 = real && ((hb[2 * tq + 8] >> grp) & 1) ? acc1[0] * p.scale_log2 : kNegInf;
    const float s3 = real && ((hb[2 * tq + 9] >> grp) & 1) ? acc1[1] * p.scale_log2 : kNegInf;
    float mt = fmaxf(fmaxf(s0, s1), fmaxf(s2, s3));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
    mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
    const float m_new = fmaxf(m_run, mt);
    float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f, alpha = 1.f;
    if (m_new != kNegInf) {
      alpha = fast_exp2(m_run - m_new);
      p0 = fast_exp2(s0 - m_new);
      p1 = fast_exp2(s1 - m_new);
      p2 = fast_exp2(s2 - m_new);
      p3 = fast_exp2(s3 - m_new);
    }
    m_run = m_new;
    l_run = l_run * alpha + (p0 + p1) + (p2 + p3);
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      o[j][0] *= alpha;
      o[j][1] *= alpha;
    }
    const uint32_t pa0 = pack_bf16(p0, p1), pa2 = pack_bf16(p2, p3);

    // ---- O += P V: lane holds dims hf*64 + grp*8 + e of tokens 2tq, 2tq+1, 2tq+8, 2tq+9
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf) {
      const int c = hf * 8 + grp;
      const int r0 = 2 * tq, r1 = 2 * tq + 1, r2 = 2 * tq + 8, r3 = 2 * tq + 9;
      const uint4 va = *reinterpret_cast<const uint4*>(Vs + r0 * ROWB + ((c ^ (r0 & 7)) << 4));
      const uint4 vb = *reinterpret_cast<const uint4*>(Vs + r1 * ROWB + ((c ^ (r1 & 7)) << 4));
      const uint4 vc = *reinterpret_cast<const uint4*>(Vs + r2 * ROWB + ((c ^ (r2 & 7)) << 4));
      const uint4 vd = *reinterpret_cast<const uint4*>(Vs + r3 * ROWB + ((c ^ (r3 & 7)) << 4));
      const uint32_t wa[4] = {va.x, va.y, va.z, va.w}, wb[4] = {vb.x, vb.y, vb.z, vb.w};
      const uint32_t wc[4] = {vc.x, vc.y, vc.z, vc.w}, wd[4] = {vd.x, vd.y, vd.z, vd.w};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t sel = (e & 1) ? 0x7632u : 0x5410u;
        const uint32_t b0 = __byte_perm(wa[e >> 1], wb[e >> 1], sel);
        const uint32_t b1 = __byte_perm(wc[e >> 1], wd[e >> 1], sel);
        float dd[4] = {o[hf * 8 + e][0], o[hf * 8 + e][1], 0.f, 0.f};
        mma_16816(dd, pa0, 0u, pa2, 0u, b0, b1);
        o[hf * 8 + e][0] = dd[0];
        o[hf * 8 + e][1] = dd[1];
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();  // the gather list and the ring are free for the next sub-chunk
  }

  // ---- merge the four warps through shared memory (reuses the ring)
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
  l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);
  __syncthreads();
  float* wm = reinterpret_cast<float*>(ring);
  float* wl = wm + kAttnWarps * GS;
  float* wo = wl + kAttnWarps * GS;
  if (grp < GS) {
    if (tq == 0) {
      wm[warp * GS + grp] = m_run;
      wl[warp * GS + grp] = l_run;
    }
#pragma unroll
    for (int hf = 0; hf < D / 64; ++hf)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        float* dst = wo + (warp * GS + grp) * D + hf * 64 + e;
        dst[(2 * tq) * 8] = o[hf * 8 + e][0];
        dst[(2 * tq + 1) * 8] = o[hf * 8 + e][1];
      }
  }
  __syncthreads();
  write_partial<D, GS>(p, b, g, split, wm, wl, wo);
}

// ---------------------------------------------------------------- fp32 / FMA
constexpr int kListBytes = ((kAttnMaxChunk + kAttnTile) * 5 + 15) / 16 * 16;
template <int D>
constexpr int attn_f32_smem_bytes() {
  return kListBytes + kAttnWarps * 8 * (D + 2) * 4;
}

// fp32 caches: one warp per token at a time, lane owns dims lane + 32 j.
template <int D, int GS>
__global__ void __launch_bounds__(kAttnThreads) attn_f32_kernel(const AttnParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int DPL = D / 32;
  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* list_idx = reinterpret_cast<int32_t*>(smem);
  uint8_t* list_hb = reinterpret_cast<uint8_t*>(list_idx + kAttnMaxChunk + kAttnTile);
  float* wm = reinterpret_cast<float*>(smem + kListBytes);
  float* wl = wm + kAttnWarps * GS;
  float* wo = wl + kAttnWarps * GS;
  __shared__ uint32_t scan_sm[32];

  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int L = p.lens[b];
  const int t0 = split * p.chunk;
  if (t0 >= L) return;
  const int t1 = min(t0 + p.chunk, L);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* Kb = reinterpret_cast<const float*>(p.k_cache);  // list entries are cache rows
  const float* Vb = reinterpret_cast<const float*>(p.v_cache);
  float q[GS][DPL], o[GS][DPL], m[GS], l[GS];
#pragma unroll
  for (int hh = 0; hh < GS; ++hh) {
    m[hh] = kNegInf;
    l[hh] = 0.f;
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      q[hh][j] = reinterpret_cast<const float*>(p.q)[((size_t)b * p.Hq + g * GS + hh) * D + lane + 32 * j];
      o[hh][j] = 0.f;
    }
  }
  for (int sc0 = t0; sc0 < t1; sc0 += kAttnMaxChunk) {
  const int n = build_union_list<GS>(p, b, g, sc0, min(sc0 + kAttnMaxChunk, t1), list_idx, list_hb, scan_sm);
  for (int i = warp; i < n; i += kAttnWarps) {
    const int t = list_idx[i];
    const uint32_t hb = list_hb[i];
    float kv[DPL], vv[DPL];
#pragma unroll
    for (int j = 0; j < DPL; ++j) {
      kv[j] = Kb[(size_t)t * D + lane + 32 * j];
      vv[j] = Vb[(size_t)t * D + lane + 32 * j];
    }
#pragma unroll
    for (int hh = 0; hh < GS; ++hh) {
      if (!((hb >> hh) & 1u)) continue;
      float dot = 0.f;
#pragma unroll
      for (int j = 0; j < DPL; ++j) dot = fmaf(q[hh][j], kv[j], dot);
#pragma unroll
      for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
      const float s = dot * p.scale_log2;
      const float mn = fmaxf(m[hh], s);
      const float alpha = exp2f(m[hh] - mn), pw = exp2f(s - mn);
      l[hh] = l[hh] * alpha + pw;
#pragma unroll
      for (int j = 0; j < DPL; ++j) o[hh][j] = o[hh][j] * alpha + pw * vv[j];
      m[hh] = mn;
    }
  }
  __syncthreads();  // the gather list is free for the next sub-chunk
  }
#pragma unroll
  for (int hh = 0; hh < GS; ++hh) {
    if (lane == 0) {
      wm[warp * GS + hh] = m[hh];
      wl[warp * GS + hh] = l[hh];
    }
#pragma unroll
    for (int j = 0; j < DPL; ++j) wo[(warp * GS + hh) * D + lane + 32 * j] = o[hh][j];
  }
  __syncthreads();
  write_partial<D, GS>(p, b, g, split, wm, wl, wo);
}

// ---------------------------------------------------------------- combine
struct CombineParams {
  const float* part_o;
  const float* part_ml;
  void* out;   // [B][Hq][D] kv dtype
  float* lse;  // [B][Hq] or nullptr
  int B, Hq, chunk, nsplit;
  int lens[kMaxBatch];
};

// fp32 log-sum-exp merge of the split partials: one CTA per (b, h).  All
// (m, l) pairs are loaded at once (one float2 each); then each of the eight
// warps sums an eighth of the splits for the whole output row (lane = D/32
// consecutive dimensions, eight split rows in flight per warp) and the
// eighths are added in shared memory.  An empty set gives out = 0 and
// lse = -inf.
constexpr int kCombineThreads = 256;
template <typename T, int D>
__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const CombineParams p) {
  pdl_wait();
  pdl_trigger();
  constexpr int DPL = D / 32;
  constexpr int NW = kCombineThreads / 32;
  __shared__ float sw[kMaxSplits];
  __shared__ float sred[NW][D];
  __shared__ float sM[NW], sS[NW];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.x;
  const int b = bh / p.Hq;
  const int L = p.lens[b];
  const int ns = (L + p.chunk - 1) / p.chunk;
  const size_t ph = (size_t)bh * p.nsplit;
  const float2* ml = reinterpret_cast<const float2*>(p.part_ml) + ph;
  float M = kNegInf;
  float2 mine[(kMaxSplits + kCombineThreads - 1) / kCombineThreads];
#pragma unroll
  for (int r = 0; r < (kMaxSplits + kCombineThreads - 1) / kCombineThreads; ++r) {
    const int sp = tid + r * kCombineThreads;
    mine[r] = sp < ns ? ml[sp] : make_float2(kNegInf, 0.f);
    M = fmaxf(M, mine[r].x);
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (lane == 0) sM[warp] = M;
  __syncthreads();
  M = sM[0];
#pragma unroll
  for (int w = 1; w < NW; ++w) M = fmaxf(M, sM[w]);
  float lsum = 0.f;
#pragma unroll
  for (int r = 0; r < (kMaxSplits + kCombineThreads - 1) / kCombineThreads; ++r) {
    const int sp = tid + r * kCombineThreads;
    if (sp < ns) {
      const float f = (M == kNegInf || mine[r].x == kNegInf) ? 0.f : exp2f(mine[r].x - M);
      sw[sp] = f;
      lsum += f * mine[r].y;
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
  if (lane == 0) sS[warp] = lsum;
  __syncthreads();
  lsum = 0.f;
#pragma unroll
  for (int w = 0; w < NW; ++w) lsum += sS[w];
  float acc[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) acc[i] = 0.f;
  const float* po = p.part_o + ph * D + lane * DPL;
#pragma unroll 8
  for (int sp = warp; sp < ns; sp += NW) {
    const float w = sw[sp];
    if constexpr (DPL == 4) {
      const float4 v = *reinterpret_cast<const float4*>(po + (size_t)sp * D);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
      acc[2] += w * v.z;
      acc[3] += w * v.w;
    } else {
      const float2 v = *reinterpret_cast<const float2*>(po + (size_t)sp * D);
      acc[0] += w * v.x;
      acc[1] += w * v.y;
    }
  }
#pragma unroll
  for (int i = 0; i < DPL; ++i) sred[warp][lane * DPL + i] = acc[i];
  __syncthreads();
  const float inv = M == kNegInf ? 0.f : 1.f / lsum;
  for (int d = tid; d < D; d += kCombineThreads) {
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < NW; ++w) o += sred[w][d];
    reinterpret_cast<T*>(p.out)[(size_t)bh * D + d] = from_f32<T>(o * inv);
  }
  if (p.lse != nullptr && tid == 0) p.lse[bh] = M == kNegInf ? kNegInf : (M + log2f(lsum)) * 0.69314718055994531f;
}

}  // namespace tb
