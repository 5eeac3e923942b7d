// butler_score: s[b][h][t] = q_hat[b][h] . K_imp[b][g(h)][t] for every cached
// token t < len[b] (model card "Meta-Llama-3.1-8B-Instruct-Butler", section
// "Method": a consumer scores every cached token with its producer's
// importance query, slot (l - 1) mod G).
//
// HBM stream over K_imp (d' fp32 = 64 or 128 bytes per token and KV head),
// read once per KV head and shared by the Hq/Hkv query heads of the group.
// Persistent CTAs (one per SM) walk a contiguous range of 256-token tiles;
// each tile is brought in by one TMA 2-D load (128B/64B swizzle, so the
// thread-per-token reads below are bank-conflict free) through a 4-stage
// mbarrier ring.  Optionally accumulates, per query-head row, the histogram
// of the top 11 bits of the order key over the candidate range
// [sink, len - window): the first radix digit of the selection.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kScoreTile = 256;   // tokens per TMA box / threads per CTA
constexpr int kScoreStages = 4;
constexpr int kHistBins = 2048;   // 11-bit first digit

struct ScoreParams {
  const void* q_imp;  // [(B*Hq)][G][1][d'] of the producer, kv dtype
  float* scores;      // [B][Hq][max_len]
  uint32_t* hist;     // [B*Hq][2048] or nullptr
  uint32_t* status;
  int G, slot, Hq, Hkv, max_len;
  int sink, window;
  int total_tiles;
  int tile_base[kMaxBatch + 1];  // prefix over b of Hkv * ceil(len[b] / 256)
  int lens[kMaxBatch];
};

template <int DIMP>
__device__ __forceinline__ int swz_offset(int row, int j) {
  // byte offset of the j-th 16-byte piece of `row` inside a TMA-swizzled box
  const int o = row * (DIMP * 4) + j * 16;
  constexpr int mask = DIMP == 32 ? 7 : 3;  // 128B or 64B swizzle
  return o ^ (((o >> 7) & mask) << 4);
}

template <typename T, int DIMP, int GS, bool HIST>
__global__ void __launch_bounds__(kScoreTile, 1)
    score_kernel(const __grid_constant__ CUtensorMap kimp_map, const ScoreParams p) {
  constexpr int STAGE_BYTES = kScoreTile * DIMP * 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kScoreStages * STAGE_BYTES);
  uint32_t* hist = reinterpret_cast<uint32_t*>(full + kScoreStages);  // [GS][2048] when HIST
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int begin = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
  const int end = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);
  const int n = end - begin;
  if (n <= 0) return;

  if (tid == 0) {
    for (int s = 0; s < kScoreStages; ++s) mbar_init(&full[s], 1);
    mbar_fence_init();
    s_abort = 0;
  }
  if (HIST)
    for (int i = tid; i < GS * kHistBins; i += kScoreTile) hist[i] = 0;
  __syncthreads();

  // tile gt -> (b, g, tile); b advances monotonically over the range
  auto decode = [&](int gt, int& b, int& g, int& tile) {
    while (gt >= p.tile_base[b + 1]) ++b;
    const int nt = (p.lens[b] + kScoreTile - 1) / kScoreTile;
    const int local = gt - p.tile_base[b];
    g = local / nt;
    tile = local - g * nt;
  };
  auto issue = [&](int i) {
    int b = 0, g, tile;
    decode(begin + i, b, g, tile);
    const int st = i % kScoreStages;
    mbar_expect_tx(&full[st], STAGE_BYTES);
    tma_load_2d(smem + st * STAGE_BYTES, &kimp_map, 0, (b * p.Hkv + g) * p.max_len + tile * kScoreTile, &full[st]);
  };
  if (tid == 0)
    for (int i = 0; i < min(kScoreStages, n); ++i) issue(i);

  float q[GS][DIMP];
  int cur_b = -1, cur_g = -1, b = 0;
  for (int i = 0; i < n; ++i) {
    int g, tile;
    decode(begin + i, b, g, tile);
    if (b != cur_b || g != cur_g) {
      if (HIST && cur_b >= 0) {  // flush the previous group's histograms
        __syncthreads();
        for (int e = tid; e < GS * kHistBins; e += kScoreTile) {
          const uint32_t c = hist[e];
          if (c) {
            atomicAdd(&p.hist[((size_t)cur_b * p.Hq + cur_g * GS + e / kHistBins) * kHistBins + e % kHistBins], c);
            hist[e] = 0;
          }
        }
      }
      cur_b = b;
      cur_g = g;
      const T* qi = reinterpret_cast<const T*>(p.q_imp);
#pragma unroll
      for (int hh = 0; hh < GS; ++hh) {
        const T* row = qi + (((size_t)b * p.Hq + g * GS + hh) * p.G + p.slot) * DIMP;
#pragma unroll
        for (int j = 0; j < DIMP; ++j) q[hh][j] = to_f32(row[j]);
      }
    }
    const int st = i % kScoreStages;
    if (!mbar_wait(&full[st], (i / kScoreStages) & 1)) s_abort = i + 1;
    __syncthreads();
    if (s_abort) break;

    const uint8_t* sb = smem + st * STAGE_BYTES;
    float kv[DIMP];
#pragma unroll
    for (int j = 0; j < DIMP / 4; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(sb + swz_offset<DIMP>(tid, j));
      kv[4 * j] = v.x;
      kv[4 * j + 1] = v.y;
      kv[4 * j + 2] = v.z;
      kv[4 * j + 3] = v.w;
    }
    const int L = p.lens[b];
    const int t = tile * kScoreTile + tid;
#pragma unroll
    for (int hh = 0; hh < GS; ++hh) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < DIMP; ++j) acc = fmaf(q[hh][j], kv[j], acc);
      if (t < L) p.scores[((size_t)b * p.Hq + g * GS + hh) * p.max_len + t] = acc;
      if (HIST) {
        const bool cand = t >= p.sink && t < L - p.window;
        const uint32_t bin = cand ? (order_key(acc) >> 21) : 0xFFFFFFFFu;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (cand && (threadIdx.x & 31) == __ffs(peers) - 1) atomicAdd(&hist[hh * kHistBins + bin], __popc(peers));
      }
    }
    __syncthreads();  // stage fully consumed
    if (tid == 0 && i + kScoreStages < n) issue(i + kScoreStages);
  }

  if (s_abort) {
    if (tid == 0) {
      atomicOr(p.status, TB_DEV_ERR_TIMEOUT);
      // wait (bounded) for the loads still in flight before leaving
      const int i0 = s_abort - 1;
      for (int j = i0; j < n && j < i0 + kScoreStages; ++j)
        (void)mbar_wait(&full[j % kScoreStages], (j / kScoreStages) & 1);
    }
    return;
  }
  if (HIST) {
    __syncthreads();
    for (int e = tid; e < GS * kHistBins; e += kScoreTile) {
      const uint32_t c = hist[e];
      if (c) atomicAdd(&p.hist[((size_t)cur_b * p.Hq + cur_g * GS + e / kHistBins) * kHistBins + e % kHistBins], c);
    }
  }
}

// zero the first-digit histograms before a fused score pass
__global__ void zero_u32_kernel(uint32_t* p, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0;
}

}  // namespace tb
