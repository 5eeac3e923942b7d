// butler_kimp_project, prefill side, on the 5th-generation tensor cores:
// K_imp = K . W_K for many cached rows (model card
// "Meta-Llama-3.1-8B-Instruct-Butler", section "Method").
//
// GEMM with M = cached rows (tiles of 128), N = d' (32 or 16), K = D (128 or
// 64), bf16 operands and fp32 accumulation in tensor memory.
//   warp 0      TMA producer: K tiles (128 rows x 64 columns per box, 128B
//               swizzle) into a 4-stage shared-memory ring of this CTA only;
//               it also writes each layer's W_K^T (N x K, K-major) into one
//               of two shared buffers in the 128B-swizzled canonical layout.
//   warp 1      one thread issues tcgen05.mma (kind::f16, M=128) per 16-wide
//               K step and commits to the ring's "empty" and the
//               accumulator's "full" mbarriers.
//   warps 2..5  epilogue: tcgen05.ld 32 lanes x d' columns each (one row per
//               thread) and plain 128-byte row stores of fp32 K_imp.
// Two accumulators in tensor memory let the epilogue of tile j overlap the
// MMAs of tile j + 1.  One launch may cover several layers (a persistent grid
// over every layer's tiles, layer by layer within a CTA, one tensor map per
// layer): W_K^T is double-buffered, the producer refills a buffer once the
// MMA issuer's commit says the MMAs of the layer before last are done, and
// the MMA issuer waits for a layer's buffer before its first MMA, so a layer
// change costs no pipeline drain.
// Every mbarrier wait is bounded; a timeout sets TB_DEV_ERR_TIMEOUT and the
// CTA winds down (tensor memory is always released).
#pragma once

#include "common.cuh"

namespace tb {

constexpr int kTcStages = 4;
constexpr int kTcRows = 128;
constexpr int kTcThreads = 192;

constexpr int kTcMaxLayers = TB_MAX_LAYERS;

struct ProjectTcParams {
  CUtensorMap kmap[kTcMaxLayers];  // per layer: K rows [B*Hkv*max_len][D], 64-column boxes of 128 rows
  const void* w_k[kTcMaxLayers];   // per layer: [D][d'] bf16
  void* kimp[kTcMaxLayers];        // per layer: [B][Hkv][max_len/256][d'][256] (kimp_index), fp32 or bf16
  uint32_t* status;
  int max_len, start, count;
  int tiles_per_slab, tiles_per_layer, total_tiles, n_layers;
  int kimp_bf16;    // store K_imp rounded to bf16
};

__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t smem_addr) {
  // K-major, 128B swizzle: 8-row core-matrix groups 1024 B apart (SBO), LBO
  // unused (1), descriptor version 1, layout type 2 (SWIZZLE_128B).
  uint64_t d = 0;
  d |= (uint64_t)((smem_addr & 0x3FFFF) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

template <int N>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&v)[N]);
template <>
__device__ __forceinline__ void tmem_ld_row<32>(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
template <>
__device__ __forceinline__ void tmem_ld_row<16>(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

template <int D>
constexpr int project_tc_smem_bytes() {
  return 1024 + kTcStages * kTcRows * D * 2 + 2 * 4096 * (D / 64) /*two W^T buffers of <= 32 rows x 128 B per atom*/ +
         256;
}

template <int D, int DIMP>
__global__ void __launch_bounds__(kTcThreads, 1)
    project_tc_kernel(const __grid_constant__ ProjectTcParams p) {
  static_assert(D == 64 || D == 128, "head dim");
  static_assert(DIMP == 16 || DIMP == 32, "importance dim");
  constexpr int ATOMS = D / 64;                       // 128-byte swizzle atoms along K
  constexpr int A_ATOM = kTcRows * 128;               // bytes of one atom column of an A tile
  constexpr int A_STAGE = ATOMS * A_ATOM;
  constexpr int B_ATOM = DIMP * 128;
  constexpr int KSTEPS = D / 16;
  constexpr int TMEM_COLS = 2 * DIMP < 32 ? 32 : 2 * DIMP;
  // kind::f16 instruction descriptor: D fp32, A/B bf16, K-major, N = DIMP, M = 128
  constexpr uint32_t IDESC = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(DIMP >> 3) << 17) |
                             ((uint32_t)(kTcRows >> 4) << 24);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* A = smem;
  uint8_t* Bt = smem + kTcStages * A_STAGE;  // two W^T buffers of ATOMS * 4096 bytes
  static_assert(B_ATOM <= 4096, "W^T atom");
  uint64_t* full = reinterpret_cast<uint64_t*>(Bt + 2 * ATOMS * 4096);
  uint64_t* empty = full + kTcStages;
  uint64_t* accf = empty + kTcStages;
  uint64_t* acce = accf + 2;
  uint64_t* wfull = acce + 2;   // W^T buffer written (producer arrives)
  uint64_t* wfree = wfull + 2;  // MMAs reading a W^T buffer completed (MMA commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(wfree + 2);
  __shared__ int s_abort_store, s_issued_store, s_consumed_store;
  volatile int* s_abort = &s_abort_store;      // set by any role, polled by all
  volatile int* s_issued = &s_issued_store;    // TMA loads issued (producer)
  volatile int* s_consumed = &s_consumed_store;  // stages consumed by the MMA issuer

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---- set-up: barriers, tensor memory, W_K^T in the swizzled K-major layout
  if (tid == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&accf[a], 1);
      mbar_init(&acce[a], 4);
      mbar_init(&wfull[a], 1);
      mbar_init(&wfree[a], 1);
    }
    mbar_fence_init();
    *s_abort = 0;
    *s_issued = 0;
    *s_consumed = 0;
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int ntiles = p.total_tiles > (int)blockIdx.x
                         ? (p.total_tiles - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x
                         : 0;
  // tile j of this CTA: K rows [t0, t0 + valid) of slab (b * Hkv + g) of
  // layer `layer`; row0 is the same row in the flattened [B*Hkv*max_len][D]
  // view used by TMA.  A CTA's tiles come layer by layer.
  auto layer_of = [&](int j) { return (int)((blockIdx.x + (long long)j * gridDim.x) / p.tiles_per_layer); };
  auto tile_of = [&](int j, int& row0, int& valid, int& slab, int& t0) {
    const int i = (int)((blockIdx.x + (long long)j * gridDim.x) % p.tiles_per_layer);
    slab = i / p.tiles_per_slab;
    const int tt = i % p.tiles_per_slab;
    t0 = p.start + tt * kTcRows;
    row0 = slab * p.max_len + t0;
    valid = min(kTcRows, p.count - tt * kTcRows);
  };

  if (warp == 0) {  // ---- producer warp: W^T buffers (all lanes), TMA loads (lane 0)
    int cur = -1, li = -1;  // current layer, its index among this CTA's layers
    for (int j = 0; j < ntiles; ++j) {
      if (__any_sync(0xffffffffu, *s_abort != 0)) break;
      const int layer = layer_of(j);
      if (layer != cur) {  // this CTA's next layer: fill W^T buffer li & 1
        cur = layer;
        ++li;
        const int s = li & 1;
        bool ok = li < 2 || mbar_wait(&wfree[s], ((li - 2) >> 1) & 1);  // MMAs of layer li - 2 done
        if (__any_sync(0xffffffffu, !ok)) {
          *s_abort = 1;
          break;
        }
        // W [D][d'] bf16 (16-byte aligned): all of a lane's 16-byte pieces are
        // requested before any is stored, then each piece's eight elements
        // W[k][n..n+7] go to rows n..n+7 of W^T[n][k]
        const uint4* W = reinterpret_cast<const uint4*>(p.w_k[layer]);
        uint8_t* Bs = Bt + s * ATOMS * 4096;
        constexpr int PIECES = D * DIMP / 8 / 32;  // per lane
        uint4 w[PIECES];
#pragma unroll
        for (int i = 0; i < PIECES; ++i) w[i] = __ldg(W + lane + 32 * i);
#pragma unroll
        for (int i = 0; i < PIECES; ++i) {
          const int e0 = 8 * (lane + 32 * i);
          const int k = e0 / DIMP, n0 = e0 % DIMP;
          const int atom = k / 64, kc = k % 64, chunk = kc / 8;
          const uint32_t wd[4] = {w[i].x, w[i].y, w[i].z, w[i].w};
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int n = n0 + q;
            const uint16_t bits = (uint16_t)(wd[q >> 1] >> (16 * (q & 1)));
            *reinterpret_cast<uint16_t*>(Bs + atom * 4096 + n * 128 + ((chunk ^ (n & 7)) << 4) + (kc % 8) * 2) = bits;
          }
        }
        asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");  // visible to the tensor cores
        __syncwarp();
        if (lane == 0) mbar_arrive_cta(&wfull[s]);
      }
      if (lane == 0) {
        const int st = j % kTcStages;
        if (!mbar_wait(&empty[st], ((j / kTcStages) & 1) ^ 1)) {
          *s_abort = 1;
        } else {
          int row0, valid, slab, t0;
          tile_of(j, row0, valid, slab, t0);
          mbar_expect_tx(&full[st], A_STAGE);
#pragma unroll
          for (int a = 0; a < ATOMS; ++a)
            tma_load_2d(A + st * A_STAGE + a * A_ATOM, &p.kmap[layer], a * 64, row0, &full[st]);
          *s_issued = j + 1;
        }
      }
      __syncwarp();
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ---- MMA issuer
      int last = -1, cur = -1, li = -1;
      for (int j = 0; j < ntiles && !*s_abort; ++j) {
        const int st = j % kTcStages, acc = j & 1;
        const int layer = layer_of(j);
        if (layer != cur) {  // first tile of this CTA's next layer
          if (li >= 0) umma_commit(&wfree[li & 1]);  // buffer of the previous layer free once its MMAs complete
          cur = layer;
          ++li;
          if (!mbar_wait(&wfull[li & 1], (li >> 1) & 1)) {
            *s_abort = 1;
            break;
          }
        }
        if (!mbar_wait(&full[st], (j / kTcStages) & 1)) {
          *s_abort = 1;
          break;
        }
        *s_consumed = j + 1;
        if (!mbar_wait(&acce[acc], ((j >> 1) & 1) ^ 1)) {
          *s_abort = 1;
          break;
        }
        tc_fence_after();
        const uint32_t a0 = smem_u32(A + st * A_STAGE), b0 = smem_u32(Bt + (li & 1) * ATOMS * 4096);
#pragma unroll
        for (int kk = 0; kk < KSTEPS; ++kk) {
          const uint32_t off = (kk / 4) * A_ATOM + (kk % 4) * 32;
          const uint32_t boff = (kk / 4) * 4096 + (kk % 4) * 32;
          umma_f16(tmem_base + acc * DIMP, umma_desc_sw128(a0 + off), umma_desc_sw128(b0 + boff), IDESC,
                   kk > 0 ? 1u : 0u);
        }
        umma_commit(&empty[st]);
        umma_commit(&accf[acc]);
        last = j;
      }
      // the last MMAs must have completed before tensor memory is released
      if (last >= 0) (void)mbar_wait(&accf[last & 1], (last >> 1) & 1);
    }
  } else {  // ---- epilogue warps 2..5: TMEM lane quarter (warp % 4)
    const int quarter = warp & 3;
    for (int j = 0; j < ntiles; ++j) {
      const int acc = j & 1;
      bool ok = mbar_wait(&accf[acc], (j >> 1) & 1);
      if (__any_sync(0xffffffffu, !ok)) {
        *s_abort = 1;
        break;
      }
      tc_fence_after();
      float v[DIMP];
      tmem_ld_row<DIMP>(tmem_base + ((uint32_t)(quarter * 32) << 16) + acc * DIMP, v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cta(&acce[acc]);
      int row0, valid, slab, t0;
      tile_of(j, row0, valid, slab, t0);
      const int layer = layer_of(j);
      const int r = quarter * 32 + lane;
      if (r < valid) {
        // for each column the warp writes 32 consecutive tokens of one tile
        const size_t dst = kimp_index(slab, 0, t0 + r, DIMP, p.max_len);
        if (p.kimp_bf16) {
          __nv_bfloat16* k16 = reinterpret_cast<__nv_bfloat16*>(p.kimp[layer]) + dst;
#pragma unroll
          for (int c = 0; c < DIMP; ++c) k16[c * kKimpTile] = __float2bfloat16_rn(v[c]);
        } else {
          float* k32 = reinterpret_cast<float*>(p.kimp[layer]) + dst;
#pragma unroll
          for (int c = 0; c < DIMP; ++c) k32[c * kKimpTile] = v[c];
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (*s_abort && tid == 0) {
    atomicOr(p.status, TB_DEV_ERR_TIMEOUT);
    // loads issued but never consumed must land before the CTA leaves
    for (int j = *s_consumed; j < *s_issued; ++j) (void)mbar_wait(&full[j % kTcStages], (j / kTcStages) & 1);
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
}

}  // namespace tb
