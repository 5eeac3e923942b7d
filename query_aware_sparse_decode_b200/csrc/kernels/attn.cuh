// butler_sparse_attn: exact attention over a selected
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
// Both products run on mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the
// group's heads as the 8 N columns: S^T = K Q^T takes the K tile as A
// (ldmatrix), O^T = V^T P^T takes the V tile as A (ldmatrix.trans) and P^T
// as B (movmatrix.trans of the softmax fragment), so a 16-token tile costs
// D/8 mma whatever the group size.  The online softmax is kept in fp32 in
// the log2 domain.  Each CTA writes one (m, l, o) partial per head; the combine
// kernel (combine.cuh) merges the chunks with an fp32 log-sum-exp.
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
// of [t0, t1) (at most kAttnMaxChunk tokens, 64 mask words) with a head
// bitmask each; pads to a multiple of 16 with (row of t0, no head).  Warps 0
// and 1 read the words (one per lane) and scan their counts; then each thread
// expands half a word (16 tokens).
template <int GS>
__device__ __forceinline__ int build_union_list(const AttnParams& p, int b, int g, int t0, int t1, int32_t* list_idx,
                                                uint8_t* list_hb, uint32_t* scan_sm) {
  constexpr int NWM = kAttnMaxChunk / 32;
  static_assert(NWM <= 64 && kAttnThreads == 2 * NWM, "two warps hold the words; a thread expands half a word");
  __shared__ uint32_t s_u[NWM], s_excl[NWM], s_hm[GS][NWM];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwords = (t1 - t0 + 31) >> 5;
  const int w_base = t0 >> 5;
  const bool per_head = p.mask_mode == TB_MASK_PER_HEAD;
  if (warp < 2) {
    const int w = tid;
    uint32_t u = 0;
    if (w < nwords) {
      if (per_head) {
        uint32_t hm[GS];
#pragma unroll
        for (int hh = 0; hh < GS; ++hh) hm[hh] = p.mask[((size_t)b * p.Hq + g * GS + hh) * p.mask_words + w_base + w];
#pragma unroll
        for (int hh = 0; hh < GS; ++hh) {
          s_hm[hh][w] = hm[hh];
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
    const uint32_t cnt = __popc(u);
    uint32_t x = cnt;  // inclusive prefix over the warp's words
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x += y;
    }
    if (w < NWM) {
      s_u[w] = u;
      s_excl[w] = x - cnt;
    }
    if (lane == 31) scan_sm[warp] = x;
  }
  __syncthreads();
  const uint32_t tot0 = scan_sm[0];
  const int total = (int)(tot0 + (nwords > 32 ? scan_sm[1] : 0u));
  {  // thread 2w + h expands half h (16 tokens) of word w
    const int w = tid >> 1, h = tid & 1;
    if (w < nwords) {
      const uint32_t u = s_u[w];
      int pos = (int)(s_excl[w] + (w >= 32 ? tot0 : 0u) + (h ? __popc(u & 0xFFFFu) : 0));
      for (uint32_t x = h ? u >> 16 : u & 0xFFFFu; x != 0u; x &= x - 1u) {
        const int j = 16 * h + __ffs(x) - 1;
        uint32_t hb = 0xFFu;
        if (per_head) {
          hb = 0;
#pragma unroll
          for (int hh = 0; hh < GS; ++hh) hb |= ((s_hm[hh][w] >> j) & 1u) << hh;
        }
        list_idx[pos] = (int32_t)kv_row(p.kl, b, g, p.Hkv, p.max_len, t0 + 32 * w + j);  // the token's cache row
        list_hb[pos] = (uint8_t)hb;
        ++pos;
      }
    }
  }
  const int padded = (total + kAttnTile - 1) / kAttnTile * kAttnTile;
  for (int i = total + tid; i < padded; i += kAttnThreads) {
    list_idx[i] = (int32_t)kv_row(p.kl, b, g, p.Hkv, p.max_len, t0);
    list_hb[i] = 0;
  }
  __syncthreads();
  return total;
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
  constexpr int KSTEPS = D / 16;                    // k-steps of S^T = K Q^T
  constexpr int MT = D / 16;                        // m-tiles of O^T = V^T P^T
  constexpr int RPL = kAttnTile * NCH / 32;         // rows a lane copies per tensor
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

  // The tile's tokens are the M rows of S^T = K Q^T (A = the K tile, B = Q^T
  // with the group's heads as its 8 columns, heads >= GS zero) and the K
  // dimension of O^T = V^T P^T (A = the V tile read transposed, B = P^T):
  // no mma row is spent on absent heads.  B fragments of Q^T: lane (grp, tq)
  // holds head grp, dims 16kk + 2tq + {0,1} and 16kk + 8 + 2tq + {0,1}.
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
  // the two heads (columns 2tq, 2tq+1) whose scores and outputs this lane holds
  const uint32_t head_bits = ((1u << GS) - 1u) >> (2 * tq) & 3u;

  // o[mt][0..1]: dims 16mt + grp, heads 2tq + {0,1}; o[mt][2..3]: dims 16mt + grp + 8
  float o[MT][4];
#pragma unroll
  for (int j = 0; j < MT; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f};
  uint8_t* my_ring = ring + warp * kAttnStages * STAGE;
  const uint32_t ring_u32 = smem_u32(my_ring);

  // ldmatrix row addresses: lane supplies row (lane & 7) of matrix (lane >> 3).
  // K (S^T A operand): matrix j = tokens 8(j & 1) + r, piece 2kk + (j >> 1).
  // V (O^T A operand, transposed): matrix j = tokens 8(j >> 1) + r, piece 2mt + (j & 1).
  // The swizzled piece (c ^ r) of row r is (2kk ^ (c_low ^ r)) for even 2kk.
  const int lr = lane & 7, lj = lane >> 3;
  const uint32_t k_row_off = (uint32_t)((lr + 8 * (lj & 1)) * ROWB);
  const uint32_t k_x = (uint32_t)(((lj >> 1) ^ lr) << 4);
  const uint32_t v_row_off = (uint32_t)((lr + 8 * (lj >> 1)) * ROWB + kAttnTile * ROWB);
  const uint32_t v_x = (uint32_t)(((lj & 1) ^ lr) << 4);

  // gather: lane copies piece (lane % NCH) of rows (lane / NCH) * RPL + i of
  // the tile, from K and from V at the same offset
  const int g_part = lane % NCH, g_row0 = (lane / NCH) * RPL;

  // the CTA's chunk is processed in sub-chunks of up to kAttnMaxChunk tokens
  // (one gather list each); the softmax state carries across them
  for (int sc0 = t0; sc0 < t1; sc0 += kAttnMaxChunk) {
  const int n = build_union_list<GS>(p, b, g, sc0, min(sc0 + kAttnMaxChunk, t1), list_idx, list_hb, scan_sm);
  const int ntiles = n / kAttnTile + (n % kAttnTile ? 1 : 0);
  const int my_n = ntiles > warp ? (ntiles - warp + kAttnWarps - 1) / kAttnWarps : 0;

  auto issue = [&](int it) {
    const int tile = warp + it * kAttnWarps;
    uint8_t* sb = my_ring + (it % kAttnStages) * STAGE;
    int tok[RPL];
#pragma unroll
    for (int i = 0; i < RPL; i += 4) {
      const int4 t4 = *reinterpret_cast<const int4*>(list_idx + tile * kAttnTile + g_row0 + i);
      tok[i] = t4.x;
      tok[i + 1] = t4.y;
      tok[i + 2] = t4.z;
      tok[i + 3] = t4.w;
    }
#pragma unroll
    for (int i = 0; i < RPL; ++i) {
      const int row = g_row0 + i;
      const size_t off = (size_t)tok[i] * ROWB + g_part * 16;
      uint8_t* dst = sb + row * ROWB + ((g_part ^ (row & 7)) << 4);
      cp_async_16(dst, Kb + off);
      cp_async_16(dst + kAttnTile * ROWB, Vb + off);
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
    const uint32_t st = ring_u32 + (uint32_t)((it % kAttnStages) * STAGE);
    const int tile = warp + it * kAttnWarps;

    // ---- S^T = K Q^T: s[0..1] = tokens grp, s[2..3] = tokens grp + 8; heads 2tq + {0,1}
    float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < KSTEPS; ++kk) {
      uint32_t a[4];
      ldsm_x4(a, st + k_row_off + (((uint32_t)(32 * kk)) ^ k_x));
      mma_16816(s, a[0], a[1], a[2], a[3], qb[kk][0], qb[kk][1]);
    }

    // ---- masked online softmax (log2 domain) per head column
    const uint32_t hb0 = list_hb[tile * kAttnTile + grp] >> (2 * tq) & head_bits;
    const uint32_t hb1 = list_hb[tile * kAttnTile + grp + 8] >> (2 * tq) & head_bits;
    float x[4];
    x[0] = (hb0 & 1u) ? s[0] * p.scale_log2 : kNegInf;
    x[1] = (hb0 & 2u) ? s[1] * p.scale_log2 : kNegInf;
    x[2] = (hb1 & 1u) ? s[2] * p.scale_log2 : kNegInf;
    x[3] = (hb1 & 2u) ? s[3] * p.scale_log2 : kNegInf;
    float mt0 = fmaxf(x[0], x[2]), mt1 = fmaxf(x[1], x[3]);
#pragma unroll
    for (int sh = 4; sh < 32; sh <<= 1) {
      mt0 = fmaxf(mt0, __shfl_xor_sync(0xffffffffu, mt0, sh));
      mt1 = fmaxf(mt1, __shfl_xor_sync(0xffffffffu, mt1, sh));
    }
    const float mn0 = fmaxf(m_run[0], mt0), mn1 = fmaxf(m_run[1], mt1);
    // a head with no kept token so far subtracts 0: every exponent is -inf
    const float mu0 = mn0 == kNegInf ? 0.f : mn0, mu1 = mn1 == kNegInf ? 0.f : mn1;
    const float al0 = m_run[0] == mu0 ? 1.f : fast_exp2(m_run[0] - mu0);
    const float al1 = m_run[1] == mu1 ? 1.f : fast_exp2(m_run[1] - mu1);
    m_run[0] = mn0;
    m_run[1] = mn1;
    const float p0 = fast_exp2(x[0] - mu0), p1 = fast_exp2(x[1] - mu1);
    const float p2 = fast_exp2(x[2] - mu0), p3 = fast_exp2(x[3] - mu1);
    l_run[0] = l_run[0] * al0 + (p0 + p2);
    l_run[1] = l_run[1] * al1 + (p1 + p3);
    if (__any_sync(0xffffffffu, al0 != 1.f || al1 != 1.f)) {
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        o[j][0] *= al0;
        o[j][1] *= al1;
        o[j][2] *= al0;
        o[j][3] *= al1;
      }
    }
    // P (tokens x heads, C layout) -> P^T B fragments: b0 = tokens 2tq + {0,1},
    // b1 = tokens 2tq + 8 + {0,1}, head grp
    const uint32_t pb0 = movmatrix_trans(pack_bf16(p0, p1));
    const uint32_t pb1 = movmatrix_trans(pack_bf16(p2, p3));

    // ---- O^T += V^T P^T
#pragma unroll
    for (int j = 0; j < MT; ++j) {
      uint32_t a[4];
      ldsm_x4_trans(a, st + v_row_off + (((uint32_t)(32 * j)) ^ v_x));
      mma_16816(o[j], a[0], a[1], a[2], a[3], pb0, pb1);
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  __syncthreads();  // the gather list and the ring are free for the next sub-chunk
  }

  // ---- merge the four warps through shared memory (reuses the ring)
#pragma unroll
  for (int sh = 4; sh < 32; sh <<= 1) {
    l_run[0] += __shfl_xor_sync(0xffffffffu, l_run[0], sh);
    l_run[1] += __shfl_xor_sync(0xffffffffu, l_run[1], sh);
  }
  __syncthreads();
  float* wm = reinterpret_cast<float*>(ring);
  float* wl = wm + kAttnWarps * GS;
  float* wo = wl + kAttnWarps * GS;
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int h = 2 * tq + e;
    if (h < GS) {
      if (grp == 0) {
        wm[warp * GS + h] = m_run[e];
        wl[warp * GS + h] = l_run[e];
      }
      float* dst = wo + (warp * GS + h) * D;
#pragma unroll
      for (int j = 0; j < MT; ++j) {
        dst[16 * j + grp] = o[j][e];
        dst[16 * j + grp + 8] = o[j][2 + e];
      }
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

}  // namespace tb
