// butler_kimp_project, CUDA-core parts: the fused decode append (new K/V row
// + its K_imp row) and the fp32-FMA prefill projection used for fp32 caches.
// K_imp is computed in fp32 and stored as fp32, or rounded to bf16 when the
// context keeps a bf16 K_imp cache.
// Model card "Meta-Llama-3.1-8B-Instruct-Butler", section "Method":
// K_imp = K . W_K with one learned D x d' matrix per layer.
#pragma once

#include "common.cuh"

namespace tb {

struct AppendParams {
  const void* k_new;  // [B][Hkv][D]
  const void* v_new;  // [B][Hkv][D]
  void* k_cache;      // [B][Hkv][max_len][D]
  void* v_cache;
  void* kimp;         // [B][Hkv][max_len/256][d'][256] (kimp_index), fp32 or bf16
  const void* w_k;    // [D][d']
  int Hkv, D, dimp, max_len;
  int kimp_bf16;       // K_imp elements are bf16
  KvLayout kl;         // dense or paged K/V caches
  int pos[kMaxBatch];  // row written for sequence b (its length before the append)
};

// One appended row of slab (b, g), computed by a CTA of at least 128 threads
// (all of them call it: it contains barriers): writes the K and V rows, then
// K_imp[j] = sum_d K[d] W_K[d][j] in fp32 with W_K staged in shared memory;
// the first 128 threads form 128 / d' partial sums per output column (over
// D / parts dimensions each, as four interleaved chains) that are added in a
// fixed order, so the row is the same bits whichever kernel computes it.  `scratch` holds
// D * d' + 256 floats.
constexpr int kAppendScratchFloats = 128 * 32 + 256;
template <typename T>
__device__ __forceinline__ void append_row(const AppendParams& p, int g, int b, float* scratch) {
  float* wsm = scratch;             // [D][d']
  float* krow = scratch + 128 * 32;  // [D]
  float* part = krow + 128;          // [128]
  const int tid = threadIdx.x, nt = blockDim.x;
  const size_t src = ((size_t)b * p.Hkv + g) * p.D;
  const size_t row = kv_row(p.kl, b, g, p.Hkv, p.max_len, p.pos[b]);
  const T* W = reinterpret_cast<const T*>(p.w_k);
  const int nw = p.D * p.dimp;
  // the new K and V elements are requested first: their latency overlaps W_K's
  T kv = T(), vv = T();
  if (tid < p.D) {
    kv = reinterpret_cast<const T*>(p.k_new)[src + tid];
    vv = reinterpret_cast<const T*>(p.v_new)[src + tid];
  }
  constexpr int VEC = 16 / (int)sizeof(T);  // W_K staged with 16-byte loads, all in flight
  if ((reinterpret_cast<uintptr_t>(W) & 15u) == 0 && nw % VEC == 0) {
#pragma unroll 8
    for (int e = tid * VEC; e < nw; e += nt * VEC) {
      const uint4 raw = *reinterpret_cast<const uint4*>(W + e);
      const T* el = reinterpret_cast<const T*>(&raw);
#pragma unroll
      for (int i = 0; i < VEC; ++i) wsm[e + i] = to_f32(el[i]);
    }
  } else {
    for (int e = tid; e < nw; e += nt) wsm[e] = to_f32(W[e]);
  }
  if (tid < p.D) {
    reinterpret_cast<T*>(p.k_cache)[row * p.D + tid] = kv;
    reinterpret_cast<T*>(p.v_cache)[row * p.D + tid] = vv;
    krow[tid] = to_f32(kv);
  }
  __syncthreads();
  if (tid < 128) {
    const int parts = 128 / p.dimp;  // 4 (d'=32) or 8 (d'=16)
    const int j = tid % p.dimp, q = tid / p.dimp;
    const int span = p.D / parts;  // a multiple of 4
    // four interleaved chains (dimensions d = 4i + u), added in a fixed order
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    for (int d = q * span; d < (q + 1) * span; d += 4) {
      a0 = fmaf(krow[d], wsm[d * p.dimp + j], a0);
      a1 = fmaf(krow[d + 1], wsm[(d + 1) * p.dimp + j], a1);
      a2 = fmaf(krow[d + 2], wsm[(d + 2) * p.dimp + j], a2);
      a3 = fmaf(krow[d + 3], wsm[(d + 3) * p.dimp + j], a3);
    }
    part[tid] = (a0 + a1) + (a2 + a3);
  }
  __syncthreads();
  if (tid < p.dimp) {
    const int parts = 128 / p.dimp;
    float sum = 0.f;
    for (int i = 0; i < parts; ++i) sum += part[i * p.dimp + tid];
    store_kimp(p.kimp, kimp_index((size_t)b * p.Hkv + g, tid, p.pos[b], p.dimp, p.max_len), sum, p.kimp_bf16);
  }
}

// grid (Hkv, B), block 128 threads: one appended row per (b, g).
template <typename T>
__global__ void __launch_bounds__(128) append_kernel(const AppendParams p) {
  pdl_wait();
  pdl_trigger();
  __shared__ float scratch[kAppendScratchFloats];
  append_row<T>(p, blockIdx.x, blockIdx.y, scratch);
}

struct ProjectParams {
  const void* k_cache;  // [B][Hkv][max_len][D], or a page pool (KvLayout)
  void* kimp;           // [B][Hkv][max_len/256][d'][256] (kimp_index), fp32 or bf16
  const void* w_k;      // [D][d']
  int Hkv, max_len, start, count;
  KvLayout kl;
  int kimp_bf16;
};

// fp32-FMA projection of rows [start, start+count) of every (b, g).
// grid (ceil(count/32), Hkv, B), block 256: 32 rows x d' outputs per block.
constexpr int kProjRows = 32;
template <typename T, int D, int DIMP>
__global__ void __launch_bounds__(256) project_fma_kernel(const ProjectParams p) {
  constexpr int ROWS = kProjRows;
  constexpr int OUT_PER_THREAD = ROWS * DIMP / 256;  // 4 (d'=32) or 2 (d'=16)
  __shared__ float ks[ROWS][D + 1];
  __shared__ float ws[D][DIMP];
  __shared__ uint32_t krow[ROWS];  // cache rows of the block's tokens
  const int g = blockIdx.y, b = blockIdx.z, tid = threadIdx.x;
  const int r0 = p.start + blockIdx.x * ROWS;
  const T* K = reinterpret_cast<const T*>(p.k_cache);
  const T* W = reinterpret_cast<const T*>(p.w_k);
  for (int i = tid; i < D * DIMP; i += 256) ws[i / DIMP][i % DIMP] = to_f32(W[i]);
  const int rend = min(ROWS, p.start + p.count - r0);
  if (tid < ROWS) krow[tid] = tid < rend ? kv_row(p.kl, b, g, p.Hkv, p.max_len, r0 + tid) : 0u;
  __syncthreads();
  for (int i = tid; i < ROWS * D; i += 256) {
    const int r = i / D, d = i % D;
    ks[r][d] = r < rend ? to_f32(K[(size_t)krow[r] * D + d]) : 0.f;
  }
  __syncthreads();
  const int r = tid / (256 / ROWS);                          // 8 threads per row
  const int j0 = (tid % (256 / ROWS)) * OUT_PER_THREAD;
  float acc[OUT_PER_THREAD];
#pragma unroll
  for (int j = 0; j < OUT_PER_THREAD; ++j) acc[j] = 0.f;
  for (int d = 0; d < D; ++d) {
    const float kv = ks[r][d];
#pragma unroll
    for (int j = 0; j < OUT_PER_THREAD; ++j) acc[j] = fmaf(kv, ws[d][j0 + j], acc[j]);
  }
  if (r < rend) {
    const size_t slab = (size_t)b * p.Hkv + g;
#pragma unroll
    for (int j = 0; j < OUT_PER_THREAD; ++j)
      store_kimp(p.kimp, kimp_index(slab, j0 + j, r0 + r, DIMP, p.max_len), acc[j], p.kimp_bf16);
  }
}

}  // namespace tb
