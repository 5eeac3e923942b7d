// butler_score: s[b][h][t] = q_hat[b][h] . K_imp[b][g(h)][t] for every cached
// token t < len[b] (model card "Meta-Llama-3.1-8B-Instruct-Butler", section
// "Method": a consumer scores every cached token with its producer's
// importance query, slot (l - 1) mod G).
//
// HBM stream over K_imp, stored as contiguous 256-token tiles, dimension-major
// inside a tile ([b][g][t/256][j][t%256], see kimp_index), read once per KV head
// and shared by the Hq/Hkv query heads of the group.  A thread scores the
// consecutive tokens of one 16-byte load per dimension (four fp32 or eight
// bf16 K_imp values): d' independent, coalesced loads, written as batches of
// up to 16 loads ahead of their FMAs (fp32, dimension order j = 0..d'-1, the
// group's query values broadcast from shared memory) so that many loads per
// thread can be in flight; the next step's first batch is requested before
// this step's stores and histogram updates.  The FMAs run on pairs of consecutive tokens
// (fma.rn.f32x2: two independent round-to-nearest fp32 FMAs, the bits of two
// fmaf).  A CTA covers `chunk` consecutive tokens (a multiple of 32, up to
// `iters` steps of 256 threads' tokens; the launch uses 1, 2 or 4 whole
// steps, picking the count so that the grid fills the SMs).
// With GROUPED (one selection per KV group) the group's per-head fp32 scores
// are added in head order and one row per (b, g) is written instead.
// Optionally each CTA accumulates, per output row, the histogram of the
// top 11 bits of the order key over the candidate range [sink, len - window)
// (the first radix digit of the selection) and flushes it with global atomics.
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kScoreThreads = 256;
constexpr int kScoreLoadBatch = 16;  // 16-byte loads issued before their FMAs
// tokens per CTA iteration: one 16-byte load of KT elements per thread and dimension
template <typename KT>
constexpr int score_step() { return kScoreThreads * (16 / (int)sizeof(KT)); }

struct ScoreParams {
  const void* q_imp;   // [(B*Hq)][G][1][d'] of the producer, kv dtype
  const void* kimp;    // [B][Hkv][max_len/256][d'][256], KT elements
  float* scores;       // [B][Hq][max_len]
  uint32_t* hist;      // [B*Hq][2048] or nullptr
  int G, slot, Hq, Hkv, max_len;
  int sink, window;
  int chunk;           // tokens per CTA, a multiple of 32
  int iters;           // ceil(chunk / score_step<KT>()) iterations
  const uint32_t* reuse;  // [B*rows] amortised selection: rows that skip scoring, or null
  int lens[kMaxBatch];
};

// Copies of the fused first-digit histogram in shared memory: lane l adds
// into copy l % copies, so that lanes whose scores fall into the same bin
// collide less; the copies are summed when the CTA flushes.  With a bf16
// K_imp (twice the tokens per load, so twice the updates per byte) as many
// as fit 64 KB (nr rows of 2048 counters each); with an fp32 K_imp one (the
// second copy measured no faster there).
constexpr int score_hist_copies(int nr, bool kimp_bf16) {
  return !kimp_bf16 || nr >= 8 ? 1 : 8 / nr > 4 ? 4 : 8 / nr;
}
constexpr size_t score_hist_smem(int nr, bool kimp_bf16) {
  return (size_t)score_hist_copies(nr, kimp_bf16) * nr * kHistBins * 4;
}

// Packed fp32 pairs for fma.rn.f32x2.
__device__ __forceinline__ uint64_t f2_pack(uint32_t lo, uint32_t hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(lo), "r"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t ffma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// The 16 bytes of one load as fp32 pairs of consecutive tokens (bf16
// widened exactly: the low half of a word is the earlier token).
__device__ __forceinline__ void unpack16(const uint4& v, uint64_t (&x)[2]) {
  x[0] = f2_pack(v.x, v.y);
  x[1] = f2_pack(v.z, v.w);
}
__device__ __forceinline__ void unpack16(const uint4& v, uint64_t (&x)[4]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = f2_pack(w[i] << 16, w[i] & 0xFFFF0000u);
}

template <typename T, typename KT, int DIMP, int GS, bool HIST, bool GROUPED = false>
__global__ void __launch_bounds__(kScoreThreads, 2) score_kernel(const ScoreParams p) {
  constexpr int NR = GROUPED ? 1 : GS;  // output rows per (b, g): per head, or the group's sum
  constexpr int TPT = 16 / (int)sizeof(KT);  // tokens per thread and step
  constexpr int STEP = score_step<KT>();
  pdl_wait();
  pdl_trigger();
  __shared__ __align__(16) float qs[DIMP][GS];
  constexpr int HC = score_hist_copies(NR, sizeof(KT) == 2);
  extern __shared__ uint32_t hist[];  // [HC][NR][2048] when HIST
  const int chunk = blockIdx.x, g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int L = p.lens[b];
  const int t_base = chunk * p.chunk;
  if (t_base >= L) return;
  const int t_end = min(t_base + p.chunk, L);  // this CTA's tokens: [t_base, t_end)
  if (p.reuse != nullptr) {  // every row of this group reuses its cached selection: nothing to score
    const size_t r0 = GROUPED ? (size_t)b * p.Hkv + g : (size_t)b * p.Hq + g * GS;
    bool all = true;
#pragma unroll
    for (int hh = 0; hh < NR; ++hh) all = all && p.reuse[r0 + hh] != 0u;
    if (all) return;
  }
  const T* qi = reinterpret_cast<const T*>(p.q_imp);
  for (int e = tid; e < DIMP * GS; e += kScoreThreads) {
    const int j = e / GS, hh = e % GS;
    qs[j][hh] = to_f32(qi[(((size_t)b * p.Hq + g * GS + hh) * p.G + p.slot) * DIMP + j]);
  }
  if (HIST)
    for (int e = tid; e < HC * NR * kHistBins; e += kScoreThreads) hist[e] = 0;
  __syncthreads();

  const size_t slab = (size_t)b * p.Hkv + g;
  const size_t row0 = GROUPED ? (size_t)b * p.Hkv + g : (size_t)b * p.Hq + g * GS;  // first output row
  float* S = p.scores + row0 * p.max_len;
  // loads in flight per batch: 16, or 8 when the accumulators are many
  constexpr int NB0 = GS * TPT > 32 ? kScoreLoadBatch / 2 : kScoreLoadBatch;
  static_assert(DIMP % NB0 == 0 || DIMP < NB0, "d' must be a multiple of the batch");
  constexpr int NB = DIMP < NB0 ? DIMP : NB0;
  // The first batch of each iteration is requested before the previous
  // iteration's stores and histogram updates, so those overlap its latency
  // (when the accumulators are few enough to leave the registers for it).
  constexpr bool AHEAD = GS * TPT <= 32;
  uint4 v[NB];
  auto load_batch = [&](int it, int j0) {
    const int t0 = t_base + it * STEP + TPT * tid;
    if (t0 < t_end) {
      const KT* K = reinterpret_cast<const KT*>(p.kimp) + kimp_index(slab, 0, t0, DIMP, p.max_len);
#pragma unroll
      for (int jj = 0; jj < NB; ++jj) v[jj] = __ldcs(reinterpret_cast<const uint4*>(K + (j0 + jj) * kKimpTile));
    }
  };
  if (AHEAD) load_batch(0, 0);
#pragma unroll 1
  for (int it = 0; it < p.iters; ++it) {
    const int t0 = t_base + it * STEP + TPT * tid;
    if (t0 < t_end) {
      uint64_t acc2[GS][TPT / 2];  // token pairs (2u, 2u + 1)
#pragma unroll
      for (int hh = 0; hh < GS; ++hh)
#pragma unroll
        for (int u = 0; u < TPT / 2; ++u) acc2[hh][u] = 0ull;
#pragma unroll
      for (int j0 = 0; j0 < DIMP; j0 += NB) {
        if (j0 > 0 || !AHEAD) load_batch(it, j0);
#pragma unroll
        for (int jj = 0; jj < NB; ++jj) {
          uint64_t kv[TPT / 2];
          unpack16(v[jj], kv);
#pragma unroll
          for (int hh = 0; hh < GS; ++hh) {
            const uint32_t qb = __float_as_uint(qs[j0 + jj][hh]);
            const uint64_t qv = f2_pack(qb, qb);
#pragma unroll
            for (int u = 0; u < TPT / 2; ++u) acc2[hh][u] = ffma2(kv[u], qv, acc2[hh][u]);
          }
        }
      }
      if (AHEAD && it + 1 < p.iters) load_batch(it + 1, 0);
      float acc[GS][TPT];
#pragma unroll
      for (int hh = 0; hh < GS; ++hh)
#pragma unroll
        for (int u = 0; u < TPT / 2; ++u) f2_unpack(acc2[hh][u], acc[hh][2 * u], acc[hh][2 * u + 1]);
      if (GROUPED) {  // the group's row: per-head fp32 scores added in head order
#pragma unroll
        for (int u = 0; u < TPT; ++u) {
          float sum = acc[0][u];
#pragma unroll
          for (int hh = 1; hh < GS; ++hh) sum += acc[hh][u];
          acc[0][u] = sum;
        }
      }
#pragma unroll
      for (int hh = 0; hh < NR; ++hh) {
        float* srow = S + (size_t)hh * p.max_len;
        if (t0 + TPT - 1 < L) {
#pragma unroll
          for (int u = 0; u < TPT; u += 4)
            *reinterpret_cast<float4*>(srow + t0 + u) =
                make_float4(acc[hh][u], acc[hh][u + 1], acc[hh][u + 2], acc[hh][u + 3]);
        } else {
#pragma unroll
          for (int u = 0; u < TPT; ++u)
            if (t0 + u < L) srow[t0 + u] = acc[hh][u];
        }
        if (HIST) {
          uint32_t* hrow = hist + ((tid & 31) % HC * NR + hh) * kHistBins;
          if (t0 >= p.sink && t0 + TPT <= L - p.window) {  // every token of the thread a candidate
#pragma unroll
            for (int u = 0; u < TPT; ++u) atomicAdd(&hrow[order_key(acc[hh][u]) >> 21], 1u);
          } else {
#pragma unroll
            for (int u = 0; u < TPT; ++u) {
              const int t = t0 + u;
              if (t >= p.sink && t < L - p.window) atomicAdd(&hrow[order_key(acc[hh][u]) >> 21], 1u);
            }
          }
        }
      }
    }
  }
  if (HIST) {
    __syncthreads();
    for (int e = tid; e < NR * kHistBins; e += kScoreThreads) {
      uint32_t c = 0;
#pragma unroll
      for (int cp = 0; cp < HC; ++cp) c += hist[cp * NR * kHistBins + e];
      if (c) atomicAdd(&p.hist[(row0 + e / kHistBins) * kHistBins + e % kHistBins], c);
    }
  }
}

// zero the first-digit histograms before a fused score pass
__global__ void zero_u32_kernel(uint32_t* p, size_t n) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) p[i] = 0;
}

}  // namespace tb
