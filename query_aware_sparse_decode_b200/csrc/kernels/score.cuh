// butler_score: s[b][h][t] = q_hat[b][h] . K_imp[b][g(h)][t] for every cached
// token t < len[b] (model card "Meta-Llama-3.1-8B-Instruct-Butler", section
// "Method": a consumer scores every cached token with its producer's
// importance query, slot (l - 1) mod G).
//
// HBM stream over K_imp (d' fp32 = 64 or 128 bytes per token and KV head),
// read once per KV head and shared by the Hq/Hkv query heads of the group.
// Persistent CTAs (one per SM) walk a contiguous range of 256-token tiles.
// Thread 0 feeds a 4-stage ring with one TMA 2-D load per tile (128B/64B
// swizzle, so the thread-per-token reads are bank-conflict free), guarded by
// full/empty mbarriers; thread (half, t) of the 16 warps scores token t of
// every tile for one half of the group's query heads, and each warp
// releases a stage as soon as it has read it.  Optionally the warps
// accumulate, per query-head row, the
// histogram of the top 11 bits of the order key over the candidate range
// [sink, len - window): the first radix digit of the selection.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kScoreTile = 256;   // tokens per TMA box (one per consumer thread)
constexpr int kScoreStages = 4;
constexpr int kScoreThreads = 2 * kScoreTile;  // 16 warps: (token, half of the group's heads) per thread

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
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ CUtensorMap kimp_map, const ScoreParams p) {
  constexpr int STAGE_BYTES = kScoreTile * DIMP * 4;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kScoreStages * STAGE_BYTES);
  uint64_t* empty = full + kScoreStages;
  uint64_t* flush = empty + kScoreStages;                              // warp rendezvous
  uint32_t* hist = reinterpret_cast<uint32_t*>(flush + 1);             // [GS][2048] when HIST
  __shared__ int s_abort_store;
  volatile int* s_abort = &s_abort_store;

  const int tid = threadIdx.x;
  const int begin = (int)(((long long)blockIdx.x * p.total_tiles) / gridDim.x);
  const int end = (int)(((long long)(blockIdx.x + 1) * p.total_tiles) / gridDim.x);
  const int n = end - begin;
  if (n <= 0) return;

  if (tid == 0) {
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kScoreThreads / 32);  // one arrival per warp
    }
    mbar_init(flush, kScoreThreads / 32);
    mbar_fence_init();
    *s_abort = 0;
  }
  if (HIST)
    for (int i = tid; i < GS * kHistBins; i += kScoreThreads) hist[i] = 0;
  __syncthreads();

  // tile gt -> (b, g, tile); b advances monotonically over the range
  auto decode = [&](int gt, int& b, int& g, int& tile) {
    while (gt >= p.tile_base[b + 1]) ++b;
    const int nt = (p.lens[b] + kScoreTile - 1) / kScoreTile;
    const int local = gt - p.tile_base[b];
    g = local / nt;
    tile = local - g * nt;
  };
  // thread 0 feeds the ring: tile j into stage j % stages once every warp has
  // released that stage's previous tile
  int pb = 0, issued = 0;
  auto issue = [&](int j) -> bool {
    const int st = j % kScoreStages;
    if (!mbar_wait(&empty[st], ((j / kScoreStages) & 1) ^ 1)) return false;
    int g, tile;
    decode(begin + j, pb, g, tile);
    mbar_expect_tx(&full[st], STAGE_BYTES);
    tma_load_2d(smem + st * STAGE_BYTES, &kimp_map, 0, (pb * p.Hkv + g) * p.max_len + tile * kScoreTile, &full[st]);
    issued = j + 1;
    return true;
  };
  if (tid == 0)
    for (int j = 0; j < kScoreStages - 1 && j < n; ++j) (void)issue(j);

  constexpr int HPT = (GS + 1) / 2;                     // heads of this thread: the group split in two halves
  const int row = tid % kScoreTile;                      // token of the tile
  const int h0 = (tid / kScoreTile) * HPT;               // first head (within the group) of this thread
  const bool active_heads = h0 < GS;
  float q[HPT][DIMP];
  int cur_b = -1, cur_g = -1, b = 0;
  uint32_t fphase = 0;
  for (int i = 0; i < n; ++i) {
    if (tid == 0 && i + kScoreStages - 1 < n && !*s_abort)
      if (!issue(i + kScoreStages - 1)) *s_abort = 1;
    int g, tile;
    decode(begin + i, b, g, tile);
    if (b != cur_b || g != cur_g) {
      if (HIST && cur_b >= 0) {  // flush the previous group's histograms
        if (!warps_sync_bounded(flush, fphase)) *s_abort = 1;
        if (*s_abort) break;
        for (int e = tid; e < GS * kHistBins; e += kScoreThreads) {
          const uint32_t c = hist[e];
          if (c) {
            atomicAdd(&p.hist[((size_t)cur_b * p.Hq + cur_g * GS + e / kHistBins) * kHistBins + e % kHistBins], c);
            hist[e] = 0;
          }
        }
        if (!warps_sync_bounded(flush, fphase)) *s_abort = 1;
        if (*s_abort) break;
      }
      cur_b = b;
      cur_g = g;
      const T* qi = reinterpret_cast<const T*>(p.q_imp);
#pragma unroll
      for (int hh = 0; hh < HPT; ++hh) {
        const T* qrow = qi + (((size_t)b * p.Hq + g * GS + (active_heads ? h0 + hh : 0)) * p.G + p.slot) * DIMP;
#pragma unroll
        for (int j = 0; j < DIMP; ++j) q[hh][j] = to_f32(qrow[j]);
      }
    }
    const int st = i % kScoreStages;
    const bool ok = mbar_wait(&full[st], (i / kScoreStages) & 1);
    if (__any_sync(0xffffffffu, !ok)) *s_abort = 1;
    if (*s_abort) break;
    const uint8_t* sb = smem + st * STAGE_BYTES;
    float kv[DIMP];
#pragma unroll
    for (int j = 0; j < DIMP / 4; ++j) {
      const float4 v = *reinterpret_cast<const float4*>(sb + swz_offset<DIMP>(row, j));
      kv[4 * j] = v.x;
      kv[4 * j + 1] = v.y;
      kv[4 * j + 2] = v.z;
      kv[4 * j + 3] = v.w;
    }
    __syncwarp();
    if ((tid & 31) == 0) mbar_arrive_cta(&empty[st]);  // this warp is done with the stage
    if (!active_heads) continue;
    const int L = p.lens[b];
    const int t = tile * kScoreTile + row;
    const bool cand = HIST && t >= p.sink && t < L - p.window;
#pragma unroll
    for (int hh = 0; hh < HPT; ++hh) {
      float acc = 0.f;
#pragma unroll
      for (int j = 0; j < DIMP; ++j) acc = fmaf(q[hh][j], kv[j], acc);
      if (t < L) p.scores[((size_t)b * p.Hq + g * GS + h0 + hh) * p.max_len + t] = acc;
      if (cand) atomicAdd(&hist[(h0 + hh) * kHistBins + (order_key(acc) >> 21)], 1u);
    }
  }
  if (HIST && !*s_abort && warps_sync_bounded(flush, fphase)) {
    for (int e = tid; e < GS * kHistBins; e += kScoreThreads) {
      const uint32_t c = hist[e];
      if (c) atomicAdd(&p.hist[((size_t)cur_b * p.Hq + cur_g * GS + e / kHistBins) * kHistBins + e % kHistBins], c);
    }
  }
  if (tid == 0 && *s_abort) {
    atomicOr(p.status, TB_DEV_ERR_TIMEOUT);
    // loads in flight must land before the CTA leaves
    for (int j = max(0, issued - kScoreStages); j < issued; ++j)
      (void)mbar_wait(&full[j % kScoreStages], (j / kScoreStages) & 1);
  }
  __syncthreads();
}

// zero the first-digit histograms before a fused score pass
__global__ void zero_u32_kernel(uint32_t* p, size_t n) {
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0;
}

}  // namespace tb
