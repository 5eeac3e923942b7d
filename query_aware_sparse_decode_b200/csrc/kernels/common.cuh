// Device helpers shared by the decode hot-path kernels (sm_100a).
#pragma once

#include <utility>

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tb.h"

namespace tb {

constexpr int kMaxBatch = TB_MAX_BATCH;
constexpr int kHistBins = 2048;  // 11-bit first radix digit of the selection

// K_imp cache layout [B][Hkv][max_len/256][d'][256]: tiles of 256 tokens, each
// a contiguous block, dimension-major inside the tile.  Element (slab, j, t)
// with slab = b * Hkv + g:
constexpr int kKimpTile = 256;
__host__ __device__ __forceinline__ size_t kimp_index(size_t slab, int j, int t, int dimp, int max_len) {
  return slab * (size_t)max_len * dimp + (size_t)(t >> 8) * dimp * kKimpTile + (size_t)j * kKimpTile + (t & 255);
}
constexpr float kNegInf = -__builtin_huge_valf();

// ------------------------------------------------------------ K/V row layout
// Dense caches: slab (b, g) is rows [(b*Hkv + g)*max_len, ... + max_len) of
// [B][Hkv][max_len][D].  Paged caches: a pool [pages][Hkv][page_size][D] and
// a page table [B][max_pages] of page ids; token t of (b, g) is row
// (page_table[b][t / page_size]*Hkv + g)*page_size + t % page_size of the
// pool (page_size a power of two).  Rows are counted in units of D elements.
struct KvLayout {
  const int32_t* page_table;  // null: dense
  int page_size, page_shift, max_pages;
};
__device__ __forceinline__ uint32_t kv_row(const KvLayout& kl, int b, int g, int Hkv, int max_len, int t) {
  if (kl.page_table == nullptr) return ((uint32_t)b * Hkv + g) * (uint32_t)max_len + (uint32_t)t;
  const int page = kl.page_table[(size_t)b * kl.max_pages + (t >> kl.page_shift)];
  return ((uint32_t)page * Hkv + g) * (uint32_t)kl.page_size + (uint32_t)(t & (kl.page_size - 1));
}


// ------------------------------------------------------------ order keys
// Monotone map of fp32 onto uint32 (larger score -> larger key); -0.0 is
// folded onto +0.0 first so that the two compare equal.
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------ conversions
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_f32(float x);
template <>
__device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }

// two fp32 -> packed bf16x2, `lo` in the low 16 bits
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// 2^x on the special-function unit (MUFU.EX2); ex2(-inf) = 0
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// K_imp cache elements: fp32, or bf16 (the fp32 value rounded to nearest,
// ties to even) when the context stores K_imp in bf16.
__device__ __forceinline__ void store_kimp(void* base, size_t i, float v, bool bf16) {
  if (bf16)
    reinterpret_cast<__nv_bfloat16*>(base)[i] = __float2bfloat16_rn(v);
  else
    reinterpret_cast<float*>(base)[i] = v;
}

// ------------------------------------------------------------ mma.sync
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col)
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four 8x8 b16 matrices from shared memory: lanes 8j..8j+7 give the 16-byte
// row addresses of matrix j; lane (4r + c) receives row r, columns 2c and
// 2c+1 of each matrix (with .trans: column r, rows 2c and 2c+1).
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
// Transposes an 8x8 b16 matrix held one register per lane in the layout above.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;\n" : "=r"(y) : "r"(x));
  return y;
}

// ------------------------------------------------------------ cp.async (LDGSTS)
// Programmatic dependent launch.  Every kernel of the decode chain starts with
// pdl_wait() (returns once the stream's preceding kernel has completed and its
// writes are visible; a no-op for a normal launch) and then pdl_trigger()
// (lets the next kernel be scheduled onto SMs this grid frees), so the launch
// latency and prologue of kernel i+1 overlap the tail of kernel i.  All CTAs
// execute the wait before any global access or early return, which keeps the
// order of every kernel pair in the stream transitive.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void cp_async_16(void* smem, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem)), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// ------------------------------------------------------------ mbarrier + TMA
// Every wait is bounded in time: about one second of SM clocks, after which
// the caller records TB_DEV_ERR_TIMEOUT and leaves.
constexpr long long kWaitCycles = 2000000000LL;

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// true when the phase with `parity` completed, false after the time limit
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit = kWaitCycles) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > limit) return false;
  }
  return true;
}

__device__ __forceinline__ void mbar_arrive_cta(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}
// Bounded rendezvous of `nwarps` warps on an mbarrier initialised with count
// nwarps: lane 0 of each warp arrives, every lane waits for the phase to
// complete.  `phase` is the caller's running phase counter.  Returns false
// after the time limit.
__device__ __forceinline__ bool warps_sync_bounded(uint64_t* bar, uint32_t& phase) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive_cta(bar);
  const bool ok = mbar_wait(bar, phase & 1);
  ++phase;
  return __all_sync(0xffffffffu, ok);
}
// 2-D tiled TMA load into this CTA's shared memory only, completing on `bar`
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::"r"(
          smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// Lanes below this one in the warp, as a bit mask.
__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

// Drops the 128-byte line at p (128-byte aligned) from L2 without writing it
// back: for intermediates that no later kernel reads, so that their dirty
// lines do not cost HBM write bandwidth when they are evicted.
__device__ __forceinline__ void discard_l2(const void* p) {
  asm volatile("discard.global.L2 [%0], 128;" ::"l"(__cvta_generic_to_global(p)) : "memory");
}

// ------------------------------------------------------------ block scans
// Exclusive prefix sum over a block of NT threads (NT a multiple of 32,
// NT <= 1024).  `sm` holds >= 32 words.  Every thread must call it.
template <int NT>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t& total, uint32_t* sm) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sm[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = lane < NW ? sm[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NW) sm[lane] = w;
  }
  __syncthreads();
  const uint32_t base = warp ? sm[warp - 1] : 0u;
  total = sm[NW - 1];
  __syncthreads();
  return base + x - v;
}

// Exclusive prefix sums of two fields at once (same contract as
// block_excl_scan; `sm` holds >= 32 uint2).
template <int NT>
__device__ __forceinline__ uint2 block_excl_scan2(uint2 v, uint2& total, uint2* sm) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint2 x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t a = __shfl_up_sync(0xffffffffu, x.x, o), c = __shfl_up_sync(0xffffffffu, x.y, o);
    if (lane >= o) {
      x.x += a;
      x.y += c;
    }
  }
  if (lane == 31) sm[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint2 w = lane < NW ? sm[lane] : make_uint2(0u, 0u);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t a = __shfl_up_sync(0xffffffffu, w.x, o), c = __shfl_up_sync(0xffffffffu, w.y, o);
      if (lane >= o) {
        w.x += a;
        w.y += c;
      }
    }
    if (lane < NW) sm[lane] = w;
  }
  __syncthreads();
  const uint2 base = warp ? sm[warp - 1] : make_uint2(0u, 0u);
  total = sm[NW - 1];
  __syncthreads();
  return make_uint2(base.x + x.x - v.x, base.y + x.y - v.y);
}

// Host: launch a kernel with programmatic stream serialization allowed (the
// kernel must begin with pdl_wait()).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace tb

