// tb_sparse_attn_static: the sparse attention of tb_sparse_attn for callers
// that cannot allocate device memory at all.
//
// Some callers cannot call cudaMalloc (or have no allocator to hand the
// library a workspace from): code that runs where allocation is forbidden
// after start-up, such as a real-time serving loop with a fixed memory
// budget, a plug-in loaded into a host process whose device memory is owned
// by someone else, or a runtime that only exposes streams.  This entry point
// needs no tb_ctx and no workspace: the split-K partials it produces between
// its two kernels live in a file-scope static device array of fixed size
// (kStaticScratchBytes, held by every GPU that loads the library until the
// process exits).  The caller still passes the caches, queries, selection
// mask and outputs.
//
// The array is shared by every call on a device and keeps the last call's
// contents; nothing in it needs to start at zero (each split writes its whole
// partial before the merge reads it).  Calls that overlap on the GPU (other
// streams, other host threads) race on it.  The device address of the array
// is looked up once per device, on the first call made with that device
// current; make that first call before any stream capture.  The address is
// kept for the life of the process: after cudaDeviceReset (which unloads the
// library's device code) it no longer names the array, so a process that
// resets a device must not call this entry point on it again.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <mutex>

#include "kernels/attn.cuh"
#include "kernels/attn_split.cuh"
#include "kernels/combine.cuh"
#include "tb.h"

using namespace tb;

namespace {

constexpr size_t kStaticScratchBytes = TB_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_static_scratch for the current device (host code may
// not use the symbol itself as an address).
tb_status scratch_for_current_device(void** out, int* num_sms) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return TB_ERR_CUDA;
  if (cudaDeviceGetAttribute(num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return TB_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return TB_ERR_CUDA;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return TB_OK;
}

}  // namespace

extern "C" TB_API tb_status tb_sparse_attn_static(const tb_cache_view* cache, const void* q, const uint32_t* mask,
                                                  int mask_mode, void* out, float* lse, void* stream) {
  if (!cache || !q || !out || !cache->k_cache || !cache->v_cache || !cache->lens_host) return TB_ERR_INVALID_ARG;
  const int B = cache->batch, Hq = cache->n_q_heads, Hkv = cache->n_kv_heads, D = cache->head_dim;
  const int max_len = cache->max_len;
  if (B < 1 || B > TB_MAX_BATCH || Hq < 1 || Hkv < 1 || Hq % Hkv) return TB_ERR_SHAPE;
  const int gs = Hq / Hkv;
  if ((gs != 1 && gs != 2 && gs != 4 && gs != 8) || (D != 64 && D != 128)) return TB_ERR_UNSUPPORTED;
  if (max_len < 256 || max_len % 256) return TB_ERR_SHAPE;
  // the gather lists hold 32-bit cache row numbers, and score-sized row
  // offsets must fit 40 bits: the same limits as a context's configuration
  if ((long long)B * Hkv * max_len >= (1LL << 31)) return TB_ERR_SHAPE;
  if ((long long)B * Hq * max_len >= (1LL << 40)) return TB_ERR_SHAPE;
  if (cache->kv_dtype != TB_BF16 && cache->kv_dtype != TB_F32) return TB_ERR_INVALID_ARG;
  if (mask_mode != TB_MASK_PER_HEAD && mask_mode != TB_MASK_SHARED && mask_mode != TB_MASK_DENSE &&
      mask_mode != TB_MASK_GROUP)
    return TB_ERR_INVALID_ARG;
  if (mask_mode != TB_MASK_DENSE && !mask) return TB_ERR_INVALID_ARG;
  int maxL = 0;
  for (int b = 0; b < B; ++b) {
    if (cache->lens_host[b] < 0 || cache->lens_host[b] > max_len) return TB_ERR_CAPACITY;
    maxL = std::max(maxL, cache->lens_host[b]);
  }

  void* scratch = nullptr;
  int num_sms = 0;
  tb_status s = scratch_for_current_device(&scratch, &num_sms);
  if (s != TB_OK) return s;

  // the chunking rule of tb_sparse_attn (attn_split)
  int chunk = 0, nsplit = 0;
  if (!attn_split(num_sms, B * Hkv, maxL, &chunk, &nsplit)) return TB_ERR_UNSUPPORTED;
  const size_t part_o_floats = (size_t)B * Hq * nsplit * D;
  const size_t part_ml_floats = (size_t)B * Hq * nsplit * 2;
  if ((part_o_floats + part_ml_floats) * sizeof(float) > kStaticScratchBytes) return TB_ERR_CAPACITY;

  AttnParams p{};
  p.k_cache = cache->k_cache;
  p.v_cache = cache->v_cache;
  p.q = q;
  p.mask = mask;
  p.part_o = static_cast<float*>(scratch);
  p.part_ml = p.part_o + part_o_floats;
  p.status = nullptr;
  p.mask_mode = mask_mode;
  p.mask_words = max_len / 32;
  p.Hq = Hq;
  p.Hkv = Hkv;
  p.max_len = max_len;
  p.chunk = chunk;
  p.nsplit = nsplit;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)D));
  for (int b = 0; b < B; ++b) p.lens[b] = cache->lens_host[b];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  dim3 grid(nsplit, Hkv, B);
#define TB_STATIC_ATTN_CASE(DV, GSV)                                                          \
  if (D == DV && gs == GSV) {                                                                 \
    if (cache->kv_dtype == TB_BF16) {                                                         \
      auto k = attn_bf16_kernel<DV, GSV>;                                                     \
      const int smem = attn_bf16_smem_bytes<DV>();                                            \
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
        return TB_ERR_CUDA;                                                                   \
      launch_pdl(k, grid, dim3(kAttnThreads), smem, st, p);                                   \
    } else {                                                                                  \
      auto k = attn_f32_kernel<DV, GSV>;                                                      \
      const int smem = attn_f32_smem_bytes<DV>();                                             \
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
        return TB_ERR_CUDA;                                                                   \
      launch_pdl(k, grid, dim3(kAttnThreads), smem, st, p);                                   \
    }                                                                                         \
  } else
  TB_STATIC_ATTN_CASE(128, 4) TB_STATIC_ATTN_CASE(128, 2) TB_STATIC_ATTN_CASE(128, 1) TB_STATIC_ATTN_CASE(128, 8)
  TB_STATIC_ATTN_CASE(64, 4) TB_STATIC_ATTN_CASE(64, 2) TB_STATIC_ATTN_CASE(64, 1) TB_STATIC_ATTN_CASE(64, 8)
  return TB_ERR_UNSUPPORTED;
#undef TB_STATIC_ATTN_CASE
  if (cudaGetLastError() != cudaSuccess) return TB_ERR_CUDA;

  CombineParams cp{};
  cp.part_o = p.part_o;
  cp.part_ml = p.part_ml;
  cp.out = out;
  cp.lse = lse;
  cp.B = B;
  cp.Hq = Hq;
  cp.chunk = chunk;
  cp.nsplit = nsplit;
  for (int b = 0; b < B; ++b) cp.lens[b] = cache->lens_host[b];
  const unsigned cgrid = (unsigned)(B * Hq);
  if (cache->kv_dtype == TB_BF16) {
    if (D == 128) launch_pdl(combine_kernel<__nv_bfloat16, 128>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
    else launch_pdl(combine_kernel<__nv_bfloat16, 64>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
  } else {
    if (D == 128) launch_pdl(combine_kernel<float, 128>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
    else launch_pdl(combine_kernel<float, 64>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
  }
  return cudaGetLastError() == cudaSuccess ? TB_OK : TB_ERR_CUDA;
}
