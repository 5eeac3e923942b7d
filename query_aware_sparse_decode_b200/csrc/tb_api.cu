// C ABI of the TokenButler decode-step hot path (declared in include/tb.h):
// host-side validation, workspace layout, per-layer bookkeeping and
// stream-ordered kernel launches.  No device memory is allocated here.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>

#include "kernels/attn.cuh"
#include "kernels/attn_split.cuh"
#include "kernels/combine.cuh"
#include "kernels/index_mask.cuh"
#include "kernels/common.cuh"
#include "kernels/kimp.cuh"
#include "kernels/prefill.cuh"
#include "kernels/reuse.cuh"
#include "kernels/project_tc.cuh"
#include "kernels/score.cuh"
#include "kernels/select.cuh"
#include "kernels/select_cluster.cuh"
#include "kernels/shard.cuh"
#include "kernels/softvote.cuh"
#include "tb.h"

using namespace tb;

namespace {

struct LayerState {
  void* k = nullptr;
  void* v = nullptr;
  void* kimp = nullptr;  // fp32 or bf16 (cfg.kimp_bf16)
  const void* wk = nullptr;
  bool bound = false;
  CUtensorMap k_map;  // bf16 caches: K rows, 64-column boxes of 128 rows, 128B swizzle
  int lens[TB_MAX_BATCH];
  KvLayout kl{};       // dense (page_table null) or paged K/V caches
  // selection cache (amortised selection), caller-owned, or null
  float* sc_q = nullptr;        // [B*rows][d'] importance query of the cached set
  int32_t* sc_len = nullptr;    // [B*rows] length at which it was selected (0: empty)
  uint32_t* sc_mask = nullptr;  // [B*rows][max_len/32] the cached mask
  // sequence sharding: this layer's caches hold global tokens [shard_t0, shard_t0 + lens[b])
  bool shard_on = false;
  int shard_t0 = 0;
  int glen[TB_MAX_BATCH];
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct WsLayout {
  size_t status, hist, ccount, kcount, hist2, ctot, hist_end, cslot, rowinfo, cand, scores, mask, part_o, part_ml, votes,
      vstats, reuse, total;
  int max_splits;
};

WsLayout layout_of(const tb_config& c) {
  WsLayout w{};
  const size_t B = c.batch, Hq = c.n_q_heads, Lm = c.max_len;
  w.max_splits = (int)std::min<size_t>((Lm + 31) / 32, kMaxSplits);  // attention splits: 32-token chunks at least
  size_t off = 0;
  w.status = off;  off += align256(256);
  w.hist = off;    off += B * Hq * kHistBins * 4;        // first-digit histograms, then
  w.ccount = off;  off += align256(B * Hq * 4);          // candidate counters, kept-token
  w.kcount = off;  off += align256(B * Hq * 4);          // counters and the single-row
  w.hist2 = off;   off += align256(B * kHistBins * 4);   // second-digit histograms and the
  w.ctot = off;    off += align256(B * Hq * (size_t)kClTotWords * 4);  // cluster selection's totals
  w.hist_end = off;                                      // (zeroed together)
  w.cslot = off;   off += align256(B * Hq * (size_t)kClSlotWords * 4);  // cluster selection's per-CTA counts
  w.rowinfo = off; off += align256(B * Hq * 16);
  w.cand = off;    off += align256(B * Hq * (size_t)kSelCap * 8);
  w.scores = off;  off += align256(B * Hq * Lm * 4);
  w.mask = off;    off += align256(B * Hq * (Lm / 32) * 4);
  w.part_o = off;  off += align256(B * Hq * (size_t)w.max_splits * c.head_dim * 4);
  w.part_ml = off; off += align256(B * Hq * (size_t)w.max_splits * 2 * 4);
  w.votes = off;   off += align256(B * Lm * 4);
  w.vstats = off;  off += align256(B * Hq * ((Lm + kVoteMinChunk - 1) / kVoteMinChunk) * 2 * 4);
  w.reuse = off;   off += align256(B * Hq * 4);         // per-row reuse decisions of the step
  w.total = off;
  return w;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

struct tb_ctx {
  tb_config cfg;
  int device = 0;
  int num_sms = 148;
  char* ws = nullptr;
  WsLayout lay;
  uint32_t* status = nullptr;
  uint32_t* hist = nullptr;
  uint32_t* ccount = nullptr;
  uint32_t* kcount = nullptr;
  uint32_t* hist2 = nullptr;
  uint32_t* cand = nullptr;
  uint4* rowinfo = nullptr;
  float* scores = nullptr;
  uint32_t* mask = nullptr;
  float* part_o = nullptr;
  float* part_ml = nullptr;
  float* votes = nullptr;
  float* vstats = nullptr;
  bool hist_clean = false;  // histograms and counters known to be zero (cleared by the last selection)
  // resident clusters of 1, 2, 4, 8, 16 CTAs of the selection kernel (0: not launchable), for its
  // 512-thread and its 1024-thread CTAs
  int cluster_active[5] = {};
  int cluster_active_few[5] = {};
  uint32_t* ctot = nullptr;
  uint32_t* cslot = nullptr;
  uint32_t* reuse = nullptr;
  float reuse_tau = 0.f;     // amortised selection: cosine threshold,
  int reuse_interval = 0;    // at most this many tokens since the cached selection (0: off),
  int reuse_radius = 0;      // neighbours t +- 1..r of the cached top-k kept as well
  cudaEvent_t trace[6] = {};
  bool tracing = false;
  unsigned long long launches = 0;
  LayerState layers[TB_MAX_LAYERS];
};

static void trace_point(tb_ctx* ctx, int i, cudaStream_t st) {
  if (ctx->tracing) cudaEventRecord(ctx->trace[i], st);
}

// ------------------------------------------------------------------ validation
static tb_status check_config(const tb_config* c) {
  if (!c) return TB_ERR_INVALID_ARG;
  if (c->n_layers < 1 || c->n_layers > TB_MAX_LAYERS) return TB_ERR_SHAPE;
  if (c->batch < 1 || c->batch > TB_MAX_BATCH) return TB_ERR_SHAPE;
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads) return TB_ERR_SHAPE;
  const int gs = c->n_q_heads / c->n_kv_heads;
  if (gs != 1 && gs != 2 && gs != 4 && gs != 8) return TB_ERR_UNSUPPORTED;
  if (c->head_dim != 64 && c->head_dim != 128) return TB_ERR_UNSUPPORTED;
  if (c->d_imp != 16 && c->d_imp != 32) return TB_ERR_UNSUPPORTED;
  if (c->producer_freq < 1) return TB_ERR_SHAPE;
  if (c->max_len < 256 || c->max_len % 256) return TB_ERR_SHAPE;
  if ((long long)c->batch * c->n_kv_heads * c->max_len >= (1LL << 31)) return TB_ERR_SHAPE;
  if ((long long)c->batch * c->n_q_heads * c->max_len >= (1LL << 40)) return TB_ERR_SHAPE;
  if (c->kv_dtype != TB_BF16 && c->kv_dtype != TB_F32) return TB_ERR_INVALID_ARG;
  if (c->keep_pct < 0 || c->keep_pct > 100 || c->sink < 0 || c->window < 0) return TB_ERR_INVALID_ARG;
  if (c->variant != TB_BUTLER && c->variant != TB_SOFTVOTE && c->variant != TB_BUTLER_GROUP)
    return TB_ERR_INVALID_ARG;
  if (c->kimp_bf16 != 0 && c->kimp_bf16 != 1) return TB_ERR_INVALID_ARG;
  if (c->kimp_bf16 && c->kv_dtype != TB_BF16) return TB_ERR_UNSUPPORTED;
  return TB_OK;
}

static tb_status check_layer(const tb_ctx* ctx, int layer) {
  if (!ctx) return TB_ERR_INVALID_ARG;
  if (layer < 0 || layer >= ctx->cfg.n_layers) return TB_ERR_INVALID_ARG;
  if (!ctx->layers[layer].bound) return TB_ERR_STATE;
  return TB_OK;
}

static tb_status cuda_status(cudaError_t e) { return e == cudaSuccess ? TB_OK : TB_ERR_CUDA; }

static int max_len_of(const LayerState& ls, int B) {
  int m = 0;
  for (int b = 0; b < B; ++b) m = std::max(m, ls.lens[b]);
  return m;
}

// How many clusters of 1, 2, 4, 8 and 16 CTAs of the cluster selection
// kernel can be resident at once on this device (0: that size cannot run).
template <int NT>
static void probe_cluster_select_nt(int (&active)[5]) {
  auto k = select_cluster_kernel<NT>;
  for (int i = 0; i < 5; ++i) active[i] = 0;
  if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, cl_smem<NT>()) != cudaSuccess ||
      cudaFuncSetAttribute(k, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return;
  }
  for (int i = 0; i < 5; ++i) {
    const int nc = 1 << i;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, 1, 1);
    cfg.blockDim = dim3(NT);
    cfg.dynamicSmemBytes = cl_smem<NT>();
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, k, &cfg) != cudaSuccess) {
      cudaGetLastError();
      clusters = 0;
    }
    active[i] = clusters;
  }
}

static void probe_cluster_select(tb_ctx* ctx) {
  probe_cluster_select_nt<kClThreadsMany>(ctx->cluster_active);
  probe_cluster_select_nt<kClThreadsFew>(ctx->cluster_active_few);
}

// ------------------------------------------------------------------ launches
// Zero the selection's histograms and candidate counters (one contiguous
// workspace range).
static void launch_zero_hist(tb_ctx* ctx, cudaStream_t st) {
  const size_t n = (ctx->lay.hist_end - ctx->lay.hist) / 4;
  launch_pdl(zero_u32_kernel, dim3((unsigned)std::min<size_t>((n + 255) / 256, 1024)), dim3(256), 0, st, ctx->hist, n);
  ++ctx->launches;
}

// Before a pass that accumulates into the histograms: zero them unless the
// previous selection's resolve kernels already did.
static void prepare_hist(tb_ctx* ctx, cudaStream_t st) {
  if (!ctx->hist_clean) launch_zero_hist(ctx, st);
  ctx->hist_clean = false;
}

static tb_status launch_score(tb_ctx* ctx, int layer, const void* q_imp, float* scores, uint32_t* hist,
                              cudaStream_t st, const uint32_t* reuse = nullptr) {
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  ScoreParams p{};
  p.q_imp = q_imp;
  p.kimp = ls.kimp;
  p.scores = scores;
  p.hist = hist;
  p.G = c.producer_freq;
  p.slot = ((layer - 1) % c.producer_freq + c.producer_freq) % c.producer_freq;
  p.Hq = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.max_len = c.max_len;
  p.sink = c.sink;
  p.window = c.window;
  p.reuse = reuse;
  for (int b = 0; b < c.batch; ++b) p.lens[b] = ls.lens[b];
  if (hist) prepare_hist(ctx, st);  // histograms and candidate counters start at zero
  const int maxL = max_len_of(ls, c.batch);
  if (maxL == 0) return cuda_status(cudaGetLastError());
  const int gs = c.n_q_heads / c.n_kv_heads;
  const bool grouped = c.variant == TB_BUTLER_GROUP;
  const size_t smem = hist ? score_hist_smem(grouped ? 1 : gs, c.kimp_bf16 != 0) : 0;
  // the most tokens per CTA (up to 4 steps) that still gives about three
  // CTAs per SM; short or small batches get one step per CTA (a grid sized
  // to whole waves of exactly balanced chunks measured no faster)
  const int step = c.kimp_bf16 ? score_step<__nv_bfloat16>() : score_step<float>();
  int iters = 4;
  while (iters > 1 && (long long)c.batch * c.n_kv_heads * ((maxL + step * iters - 1) / (step * iters)) <
                          3LL * ctx->num_sms)
    iters >>= 1;
  p.iters = iters;
  const int chunk = step * iters;
  p.chunk = chunk;
  dim3 grid((maxL + chunk - 1) / chunk, c.n_kv_heads, c.batch);
#define TB_SCORE_CASE(T, KT, DI, GSV)                                                                \
  if (c.d_imp == DI && gs == GSV) {                                                                  \
    auto k = hist ? (grouped ? score_kernel<T, KT, DI, GSV, true, true> : score_kernel<T, KT, DI, GSV, true, false>) \
                  : (grouped ? score_kernel<T, KT, DI, GSV, false, true>                             \
                             : score_kernel<T, KT, DI, GSV, false, false>);                          \
    if (hist && cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return TB_ERR_CUDA;                                                                            \
    launch_pdl(k, grid, dim3(kScoreThreads), smem, st, p);                                           \
    ++ctx->launches;                                                                                 \
    return cuda_status(cudaGetLastError());                                                          \
  }
#define TB_SCORE_CASES(T, KT)                                                                        \
  TB_SCORE_CASE(T, KT, 32, 4)                                                                        \
  TB_SCORE_CASE(T, KT, 32, 2)                                                                        \
  TB_SCORE_CASE(T, KT, 32, 1)                                                                        \
  TB_SCORE_CASE(T, KT, 32, 8)                                                                        \
  TB_SCORE_CASE(T, KT, 16, 4)                                                                        \
  TB_SCORE_CASE(T, KT, 16, 2)                                                                        \
  TB_SCORE_CASE(T, KT, 16, 1)                                                                        \
  TB_SCORE_CASE(T, KT, 16, 8)
  if (c.kv_dtype == TB_BF16 && c.kimp_bf16) {
    TB_SCORE_CASES(__nv_bfloat16, __nv_bfloat16)
  } else if (c.kv_dtype == TB_BF16) {
    TB_SCORE_CASES(__nv_bfloat16, float)
  } else {
    TB_SCORE_CASES(float, float)
  }
#undef TB_SCORE_CASES
#undef TB_SCORE_CASE
  return TB_ERR_UNSUPPORTED;
}

// Selection of every row: hist1_ready means the score kernel already built
// the first-digit histograms (and zeroed the candidate counters).
static tb_status launch_select(tb_ctx* ctx, int layer, const float* scores, bool hist1_ready, int rows,
                               int32_t* idx, int idx_cap, int32_t* count, uint32_t* mask, cudaStream_t st,
                               bool use_cache = false, bool scores_dead = false) {
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  SelectParams p{};
  p.scores = scores;
  p.hist1 = ctx->hist;
  p.hist2 = rows == 1 ? ctx->hist2 : nullptr;
  p.cand = ctx->cand;
  p.ccount = ctx->ccount;
  p.kcount = ctx->kcount;
  p.rowinfo = ctx->rowinfo;
  p.idx = idx;
  p.count = count;
  p.mask = mask != nullptr ? mask : ctx->mask;
  p.status = ctx->status;
  p.row_stride = c.max_len;
  p.rows_per_seq = rows;
  p.idx_cap = idx_cap;
  p.mask_words = c.max_len / 32;
  p.keep_pct = c.keep_pct;
  p.sink = c.sink;
  p.window = c.window;
  p.discard_scores = scores_dead ? 1 : 0;  // the decode step's workspace scores: no reader after the selection
  if (use_cache) {
    p.reuse = ctx->reuse;
    p.sc_len = ls.sc_len;
    p.sc_mask = ls.sc_mask;
    p.reuse_radius = ctx->reuse_radius;
  }
  for (int b = 0; b < c.batch; ++b) p.lens[b] = ls.lens[b];
  const int maxL = max_len_of(ls, c.batch);
  int nc = 0, chunk = 0;
  // 1024-thread CTAs when the rows' clusters fit one wave of one CTA per SM
  const long long nrows = (long long)rows * c.batch;
  bool few = cluster_select_shape(ctx->num_sms, nrows, maxL, ctx->cluster_active_few, &nc, &chunk);
  int ci = 0;
  while (few && (1 << ci) < nc) ++ci;
  few = few && nrows * nc <= ctx->num_sms && nrows <= ctx->cluster_active_few[ci];
  if (few || cluster_select_shape(ctx->num_sms, nrows, maxL, ctx->cluster_active, &nc, &chunk)) {
    // one cluster per row: one launch after the first-digit histogram
    if (!hist1_ready) {
      dim3 cgrid((std::max(maxL, 1) + kSelChunk - 1) / kSelChunk, rows, c.batch);
      prepare_hist(ctx, st);
      launch_pdl(select_hist_kernel, cgrid, dim3(kScatThreads), 0, st, p);
      ++ctx->launches;
    }
    p.ctot = ctx->ctot;
    p.cslot = ctx->cslot;
    if (few)
      launch_pdl_cluster(select_cluster_kernel<kClThreadsFew>, dim3(nc, rows, c.batch), dim3(kClThreadsFew),
                         (size_t)cl_smem<kClThreadsFew>(), st, nc, p, chunk);
    else
      launch_pdl_cluster(select_cluster_kernel<kClThreadsMany>, dim3(nc, rows, c.batch), dim3(kClThreadsMany),
                         (size_t)cl_smem<kClThreadsMany>(), st, nc, p, chunk);
    ++ctx->launches;
    const tb_status s = cuda_status(cudaGetLastError());
    if (s == TB_OK) ctx->hist_clean = true;  // CTA 0 of every row clears the row's histogram
    return s;
  }
  // rows longer than one cluster reaches: many CTAs per row scatter the
  // threshold bin's candidates, one CTA per row resolves them
  dim3 cgrid((std::max(maxL, 1) + kSelChunk - 1) / kSelChunk, rows, c.batch);
  if (!hist1_ready) {
    prepare_hist(ctx, st);
    launch_pdl(select_hist_kernel, cgrid, dim3(kScatThreads), 0, st, p);
    ++ctx->launches;
  }
  if (rows == 1) {  // one long row per sequence: split a crowded threshold bin further
    launch_pdl(select_refine_kernel, dim3((std::max(maxL, 1) + kRefChunk - 1) / kRefChunk, 1, c.batch),
               dim3(kScatThreads), 0, st, p);
    ++ctx->launches;
  }
  if (cudaFuncSetAttribute(select_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kScatSmem) !=
      cudaSuccess)
    return TB_ERR_CUDA;
  launch_pdl(select_scatter_kernel, cgrid, dim3(kScatThreads), kScatSmem, st, p);
  if (cudaFuncSetAttribute(select_resolve_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kResolveSmem) !=
      cudaSuccess)
    return TB_ERR_CUDA;
  launch_pdl(select_resolve_kernel, dim3(rows, c.batch), dim3(kSelThreads), kResolveSmem, st, p);
  ctx->launches += 2;
  const tb_status s = cuda_status(cudaGetLastError());
  if (s == TB_OK) ctx->hist_clean = true;  // every resolve CTA clears its row's state
  return s;
}

static tb_status launch_attn(tb_ctx* ctx, int layer, const void* q, const uint32_t* mask, int mode, void* out,
                             float* lse, cudaStream_t st, bool out_f32 = false) {
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  const int maxL = max_len_of(ls, c.batch);
  const int gs = c.n_q_heads / c.n_kv_heads;
  AttnParams p{};
  p.k_cache = ls.k;
  p.v_cache = ls.v;
  p.kl = ls.kl;
  p.q = q;
  p.mask = mask;
  p.part_o = ctx->part_o;
  p.part_ml = ctx->part_ml;
  p.status = ctx->status;
  p.mask_mode = mode;
  p.mask_words = c.max_len / 32;
  p.Hq = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.max_len = c.max_len;
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c.head_dim));
  for (int b = 0; b < c.batch; ++b) p.lens[b] = ls.lens[b];
  int chunk = 0;
  if (!attn_split(ctx->num_sms, c.batch * c.n_kv_heads, maxL, &chunk, &p.nsplit)) return TB_ERR_UNSUPPORTED;
  p.chunk = chunk;
  if (p.nsplit > ctx->lay.max_splits) return TB_ERR_WORKSPACE;
  {
    dim3 grid(p.nsplit, c.n_kv_heads, c.batch);
#define TB_ATTN_CASE(DV, GSV)                                                                               \
  if (c.head_dim == DV && gs == GSV) {                                                                      \
    if (c.kv_dtype == TB_BF16) {                                                                            \
      auto k = attn_bf16_kernel<DV, GSV>;                                                                   \
      const int smem = attn_bf16_smem_bytes<DV>();                                                          \
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
        return TB_ERR_CUDA;                                                                          \
      launch_pdl(k, grid, dim3(kAttnThreads), smem, st, p);                                        \
    } else {                                                                                                \
      auto k = attn_f32_kernel<DV, GSV>;                                                                    \
      const int smem = attn_f32_smem_bytes<DV>();                                                           \
      if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
        return TB_ERR_CUDA;                                                                          \
      launch_pdl(k, grid, dim3(kAttnThreads), smem, st, p);                                        \
    }                                                                                                       \
  } else
    TB_ATTN_CASE(128, 4) TB_ATTN_CASE(128, 2) TB_ATTN_CASE(128, 1) TB_ATTN_CASE(128, 8)
    TB_ATTN_CASE(64, 4) TB_ATTN_CASE(64, 2) TB_ATTN_CASE(64, 1) TB_ATTN_CASE(64, 8)
    return TB_ERR_UNSUPPORTED;
#undef TB_ATTN_CASE
    ++ctx->launches;
    tb_status s = cuda_status(cudaGetLastError());
    if (s != TB_OK) return s;
  }
  trace_point(ctx, 4, st);
  CombineParams cp{};
  cp.part_o = ctx->part_o;
  cp.part_ml = ctx->part_ml;
  cp.out = out;
  cp.lse = lse;
  cp.B = c.batch;
  cp.Hq = c.n_q_heads;
  cp.chunk = chunk;
  cp.nsplit = p.nsplit;
  for (int b = 0; b < c.batch; ++b) cp.lens[b] = ls.lens[b];
  const unsigned cgrid = (unsigned)(c.batch * c.n_q_heads);
  if (c.kv_dtype == TB_BF16 && !out_f32) {
    if (c.head_dim == 128) launch_pdl(combine_kernel<__nv_bfloat16, 128>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
    else launch_pdl(combine_kernel<__nv_bfloat16, 64>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
  } else {
    if (c.head_dim == 128) launch_pdl(combine_kernel<float, 128>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
    else launch_pdl(combine_kernel<float, 64>, dim3(cgrid), dim3(kCombineThreads), 0, st,
                    cp);
  }
  ++ctx->launches;
  trace_point(ctx, 5, st);
  return cuda_status(cudaGetLastError());
}

static tb_status launch_softvote(tb_ctx* ctx, int layer, const void* q, float* votes, uint32_t* hist,
                                cudaStream_t st) {
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  if (c.kv_dtype != TB_BF16) return TB_ERR_UNSUPPORTED;
  if (c.n_q_heads > kVoteMaxHeads) return TB_ERR_UNSUPPORTED;
  const int maxL = max_len_of(ls, c.batch);
  if (maxL == 0) return TB_OK;
  const int gs = c.n_q_heads / c.n_kv_heads;
  VoteParams p{};
  p.k_cache = ls.k;
  p.kl = ls.kl;
  p.q = q;
  p.logits = ctx->scores;
  p.stats = ctx->vstats;
  p.votes = votes;
  p.hist1 = hist;
  p.sink = c.sink;
  p.window = c.window;
  p.Hq = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.max_len = c.max_len;
  p.nchunk = (c.max_len + kVoteMinChunk - 1) / kVoteMinChunk;
  {  // about four CTAs per SM in one wave, whatever B and L
    const int nsplit = std::max(1, 4 * ctx->num_sms / (c.batch * c.n_kv_heads));
    const int chunk = ((maxL + nsplit - 1) / nsplit + 15) / 16 * 16;
    p.chunk = std::max(kVoteMinChunk, chunk);
  }
  p.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)c.head_dim));
  for (int b = 0; b < c.batch; ++b) p.lens[b] = ls.lens[b];
  dim3 grid((maxL + p.chunk - 1) / p.chunk, c.n_kv_heads, c.batch);
#define TB_VOTE_CASE(DV, GSV)                                                                 \
  if (c.head_dim == DV && gs == GSV) {                                                        \
    auto k = softvote_logits_kernel<DV, GSV>;                                                 \
    const int smem = vote_logits_smem<DV>();                                                  \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return TB_ERR_CUDA; \
    launch_pdl(k, grid, dim3(kVoteThreads), smem, st, p);                            \
  } else
  TB_VOTE_CASE(128, 4) TB_VOTE_CASE(128, 2) TB_VOTE_CASE(128, 1) TB_VOTE_CASE(128, 8)
  TB_VOTE_CASE(64, 4) TB_VOTE_CASE(64, 2) TB_VOTE_CASE(64, 1) TB_VOTE_CASE(64, 8)
  return TB_ERR_UNSUPPORTED;
#undef TB_VOTE_CASE
  ++ctx->launches;
  tb_status s = cuda_status(cudaGetLastError());
  if (s != TB_OK) return s;
  dim3 g2((maxL + kVoteReduceTok - 1) / kVoteReduceTok, c.batch);
  launch_pdl(softvote_reduce_kernel, g2, dim3(256), 0, st, p);
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}

// ------------------------------------------------------------------ C ABI
extern "C" {

TB_API tb_status tb_workspace_size(const tb_config* cfg, size_t* bytes) {
  if (!bytes) return TB_ERR_INVALID_ARG;
  tb_status s = check_config(cfg);
  if (s != TB_OK) return s;
  *bytes = layout_of(*cfg).total;
  return TB_OK;
}

TB_API tb_status tb_init(const tb_config* cfg, void* workspace, size_t ws_bytes, tb_ctx** out) {
  if (!out) return TB_ERR_INVALID_ARG;
  *out = nullptr;
  tb_status s = check_config(cfg);
  if (s != TB_OK) return s;
  const WsLayout lay = layout_of(*cfg);
  if (!workspace || ws_bytes < lay.total) return TB_ERR_WORKSPACE;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return TB_ERR_WORKSPACE;
  tb_ctx* ctx = new (std::nothrow) tb_ctx();
  if (!ctx) return TB_ERR_INVALID_ARG;
  ctx->cfg = *cfg;
  ctx->lay = lay;
  if (cudaGetDevice(&ctx->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) != cudaSuccess) {
    delete ctx;
    return TB_ERR_CUDA;
  }
  ctx->ws = static_cast<char*>(workspace);
  ctx->status = reinterpret_cast<uint32_t*>(ctx->ws + lay.status);
  ctx->hist = reinterpret_cast<uint32_t*>(ctx->ws + lay.hist);
  ctx->ccount = reinterpret_cast<uint32_t*>(ctx->ws + lay.ccount);
  ctx->kcount = reinterpret_cast<uint32_t*>(ctx->ws + lay.kcount);
  ctx->hist2 = reinterpret_cast<uint32_t*>(ctx->ws + lay.hist2);
  ctx->ctot = reinterpret_cast<uint32_t*>(ctx->ws + lay.ctot);
  ctx->cslot = reinterpret_cast<uint32_t*>(ctx->ws + lay.cslot);
  ctx->cand = reinterpret_cast<uint32_t*>(ctx->ws + lay.cand);
  ctx->rowinfo = reinterpret_cast<uint4*>(ctx->ws + lay.rowinfo);
  ctx->scores = reinterpret_cast<float*>(ctx->ws + lay.scores);
  ctx->mask = reinterpret_cast<uint32_t*>(ctx->ws + lay.mask);
  ctx->part_o = reinterpret_cast<float*>(ctx->ws + lay.part_o);
  ctx->part_ml = reinterpret_cast<float*>(ctx->ws + lay.part_ml);
  ctx->votes = reinterpret_cast<float*>(ctx->ws + lay.votes);
  ctx->vstats = reinterpret_cast<float*>(ctx->ws + lay.vstats);
  ctx->reuse = reinterpret_cast<uint32_t*>(ctx->ws + lay.reuse);
  if (cudaMemset(ctx->status, 0, sizeof(uint32_t)) != cudaSuccess) {
    delete ctx;
    return TB_ERR_CUDA;
  }
  probe_cluster_select(ctx);
  *out = ctx;
  return TB_OK;
}

TB_API tb_status tb_bind_layer(tb_ctx* ctx, int layer, void* k_cache, void* v_cache, void* kimp_cache,
                               const void* w_k) {
  if (!ctx || layer < 0 || layer >= ctx->cfg.n_layers) return TB_ERR_INVALID_ARG;
  if (!k_cache || !v_cache || !kimp_cache || !w_k) return TB_ERR_INVALID_ARG;
  if (!aligned16(k_cache) || !aligned16(v_cache) || !aligned16(kimp_cache) || !aligned16(w_k)) return TB_ERR_SHAPE;
  const tb_config& c = ctx->cfg;
  LayerState& ls = ctx->layers[layer];
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return TB_ERR_CUDA;
  cuuint32_t estride[2] = {1, 1};
  CUresult r = CUDA_SUCCESS;
  if (c.kv_dtype == TB_BF16) {
    cuuint64_t kdim[2] = {(cuuint64_t)c.head_dim, (cuuint64_t)c.batch * c.n_kv_heads * c.max_len};
    cuuint64_t kstride[1] = {(cuuint64_t)c.head_dim * 2};
    cuuint32_t kbox[2] = {64, (cuuint32_t)kTcRows};
    r = enc(&ls.k_map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, k_cache, kdim, kstride, kbox, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return TB_ERR_CUDA;
  }
  ls.k = k_cache;
  ls.v = v_cache;
  ls.kimp = kimp_cache;
  ls.wk = w_k;
  ls.kl = KvLayout{};
  std::memset(ls.lens, 0, sizeof(ls.lens));
  ls.bound = true;
  return TB_OK;
}

TB_API tb_status tb_bind_layer_paged(tb_ctx* ctx, int layer, void* k_pool, void* v_pool, int num_pages,
                                     const int32_t* page_table, int page_size, int max_pages, void* kimp_cache,
                                     const void* w_k) {
  if (!ctx || layer < 0 || layer >= ctx->cfg.n_layers) return TB_ERR_INVALID_ARG;
  if (!k_pool || !v_pool || !page_table || !kimp_cache || !w_k) return TB_ERR_INVALID_ARG;
  if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(kimp_cache) || !aligned16(w_k)) return TB_ERR_SHAPE;
  const tb_config& c = ctx->cfg;
  if (page_size < 16 || (page_size & (page_size - 1)) != 0 || num_pages < 1 || max_pages < 1) return TB_ERR_SHAPE;
  if ((long long)max_pages * page_size < c.max_len) return TB_ERR_SHAPE;
  if ((long long)num_pages * c.n_kv_heads * page_size >= (1LL << 31)) return TB_ERR_SHAPE;
  LayerState& ls = ctx->layers[layer];
  int shift = 0;
  while ((1 << shift) < page_size) ++shift;
  ls.k = k_pool;
  ls.v = v_pool;
  ls.kimp = kimp_cache;
  ls.wk = w_k;
  ls.kl = KvLayout{page_table, page_size, shift, max_pages};
  std::memset(ls.lens, 0, sizeof(ls.lens));
  ls.bound = true;
  return TB_OK;
}

TB_API tb_status tb_set_seq_lens(tb_ctx* ctx, int layer, const int32_t* lens_host) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!lens_host) return TB_ERR_INVALID_ARG;
  for (int b = 0; b < ctx->cfg.batch; ++b)
    if (lens_host[b] < 0 || lens_host[b] > ctx->cfg.max_len) return TB_ERR_CAPACITY;
  for (int b = 0; b < ctx->cfg.batch; ++b) ctx->layers[layer].lens[b] = lens_host[b];
  return TB_OK;
}

TB_API tb_status tb_get_seq_lens(const tb_ctx* ctx, int layer, int32_t* lens_host) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!lens_host) return TB_ERR_INVALID_ARG;
  for (int b = 0; b < ctx->cfg.batch; ++b) lens_host[b] = ctx->layers[layer].lens[b];
  return TB_OK;
}

TB_API tb_status tb_set_budget(tb_ctx* ctx, int keep_pct, int sink, int window) {
  if (!ctx) return TB_ERR_INVALID_ARG;
  if (keep_pct < 0 || keep_pct > 100 || sink < 0 || window < 0) return TB_ERR_INVALID_ARG;
  ctx->cfg.keep_pct = keep_pct;
  ctx->cfg.sink = sink;
  ctx->cfg.window = window;
  return TB_OK;
}

// ------------------------------------------------------------------ amortised selection
static int sel_rows(const tb_config& c) { return c.variant == TB_BUTLER_GROUP ? c.n_kv_heads : c.n_q_heads; }

struct SelCacheLayout {
  size_t q, len, mask, total;
};
static SelCacheLayout sel_cache_layout(const tb_config& c) {
  const size_t R = (size_t)c.batch * sel_rows(c);
  SelCacheLayout l{};
  size_t off = 0;
  l.q = off;    off += align256(R * c.d_imp * 4);
  l.len = off;  off += align256(R * 4);
  l.mask = off; off += align256(R * (size_t)(c.max_len / 32) * 4);
  l.total = off;
  return l;
}

TB_API tb_status tb_selection_cache_size(const tb_config* cfg, size_t* bytes) {
  if (!bytes) return TB_ERR_INVALID_ARG;
  const tb_status s = check_config(cfg);
  if (s != TB_OK) return s;
  *bytes = sel_cache_layout(*cfg).total;
  return TB_OK;
}

TB_API tb_status tb_bind_selection_cache(tb_ctx* ctx, int layer, void* cache, size_t bytes) {
  if (!ctx || layer < 0 || layer >= ctx->cfg.n_layers) return TB_ERR_INVALID_ARG;
  LayerState& ls = ctx->layers[layer];
  if (!cache) {
    ls.sc_q = nullptr;
    ls.sc_len = nullptr;
    ls.sc_mask = nullptr;
    return TB_OK;
  }
  if (ctx->cfg.variant == TB_SOFTVOTE) return TB_ERR_UNSUPPORTED;
  const SelCacheLayout l = sel_cache_layout(ctx->cfg);
  if (bytes < l.total) return TB_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(cache) & 255u) != 0) return TB_ERR_SHAPE;
  char* c = static_cast<char*>(cache);
  ls.sc_q = reinterpret_cast<float*>(c + l.q);
  ls.sc_len = reinterpret_cast<int32_t*>(c + l.len);
  ls.sc_mask = reinterpret_cast<uint32_t*>(c + l.mask);
  return TB_OK;
}

TB_API tb_status tb_copy_step_masks(tb_ctx* ctx, uint32_t* dst, size_t bytes, void* stream) {
  if (!ctx || !dst) return TB_ERR_INVALID_ARG;
  const tb_config& c = ctx->cfg;
  const int rows = c.variant == TB_SOFTVOTE ? 1 : sel_rows(c);  // soft voting: one shared set per sequence
  const size_t need = (size_t)c.batch * rows * (size_t)(c.max_len / 32) * 4;
  if (bytes < need) return TB_ERR_SHAPE;
  return cuda_status(cudaMemcpyAsync(dst, ctx->mask, need, cudaMemcpyDeviceToDevice, static_cast<cudaStream_t>(stream)));
}

TB_API tb_status tb_set_reuse(tb_ctx* ctx, float tau, int interval, int radius) {
  if (!ctx) return TB_ERR_INVALID_ARG;
  if (!(tau >= -1.f && tau <= 1.f) || interval < 0 || radius < 0 || radius > 31) return TB_ERR_INVALID_ARG;
  ctx->reuse_tau = tau;
  ctx->reuse_interval = interval;
  ctx->reuse_radius = radius;
  return TB_OK;
}

// Parameters of the append of one token per sequence at the current lengths.
static tb_status append_params(const tb_ctx* ctx, int layer, const void* k_new, const void* v_new,
                               AppendParams* p) {
  if (!k_new || !v_new) return TB_ERR_INVALID_ARG;
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  for (int b = 0; b < c.batch; ++b)
    if (ls.lens[b] >= c.max_len) return TB_ERR_CAPACITY;
  *p = AppendParams{};
  p->k_new = k_new;
  p->v_new = v_new;
  p->k_cache = ls.k;
  p->v_cache = ls.v;
  p->kimp = ls.kimp;
  p->w_k = ls.wk;
  p->kl = ls.kl;
  p->kimp_bf16 = c.kimp_bf16;
  p->Hkv = c.n_kv_heads;
  p->D = c.head_dim;
  p->dimp = c.d_imp;
  p->max_len = c.max_len;
  for (int b = 0; b < c.batch; ++b) p->pos[b] = ls.lens[b];
  return TB_OK;
}

TB_API tb_status tb_append_kv(tb_ctx* ctx, int layer, const void* k_new, const void* v_new, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  const tb_config& c = ctx->cfg;
  LayerState& ls = ctx->layers[layer];
  AppendParams p;
  s = append_params(ctx, layer, k_new, v_new, &p);
  if (s != TB_OK) return s;
  dim3 grid(c.n_kv_heads, c.batch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c.kv_dtype == TB_BF16)
    launch_pdl(append_kernel<__nv_bfloat16>, grid, dim3(128), 0, st, p);
  else
    launch_pdl(append_kernel<float>, grid, dim3(128), 0, st, p);
  ++ctx->launches;
  s = cuda_status(cudaGetLastError());
  if (s != TB_OK) return s;
  for (int b = 0; b < c.batch; ++b) ls.lens[b] += 1;
  return TB_OK;
}

// One persistent tcgen05 launch projecting rows [start, start + count) of
// every (b, KV head) of layers [first, first + n) (dense bf16 caches).
static tb_status launch_project_tc(tb_ctx* ctx, int first, int n, int start, int count, cudaStream_t st) {
  const tb_config& c = ctx->cfg;
  ProjectTcParams tp{};  // ~9 KB of kernel parameters (one tensor map per layer)
  for (int i = 0; i < n; ++i) {
    const LayerState& ls = ctx->layers[first + i];
    tp.kmap[i] = ls.k_map;
    tp.w_k[i] = ls.wk;
    tp.kimp[i] = ls.kimp;
  }
  tp.status = ctx->status;
  tp.max_len = c.max_len;
  tp.start = start;
  tp.count = count;
  tp.tiles_per_slab = (count + kTcRows - 1) / kTcRows;
  tp.tiles_per_layer = tp.tiles_per_slab * c.batch * c.n_kv_heads;
  tp.total_tiles = tp.tiles_per_layer * n;
  tp.n_layers = n;
  tp.kimp_bf16 = c.kimp_bf16;
  const int grid = std::min(tp.total_tiles, ctx->num_sms);
#define TB_TC_CASE(DV, DI)                                                              \
  if (c.head_dim == DV && c.d_imp == DI) {                                              \
    auto k = project_tc_kernel<DV, DI>;                                                 \
    const int smem = project_tc_smem_bytes<DV>();                                       \
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) \
      return TB_ERR_CUDA;                                                               \
    k<<<grid, kTcThreads, smem, st>>>(tp);                                              \
  } else
  TB_TC_CASE(128, 32) TB_TC_CASE(128, 16) TB_TC_CASE(64, 32) TB_TC_CASE(64, 16) return TB_ERR_UNSUPPORTED;
#undef TB_TC_CASE
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_project_kimp(tb_ctx* ctx, int layer, int start, int count, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  const tb_config& c = ctx->cfg;
  if (start < 0 || count < 0 || (long long)start + count > c.max_len) return TB_ERR_CAPACITY;
  if (count == 0) return TB_OK;
  const LayerState& ls = ctx->layers[layer];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c.kv_dtype == TB_BF16 && ls.kl.page_table == nullptr) return launch_project_tc(ctx, layer, 1, start, count, st);
  // fp32 caches, and paged caches of either type (a TMA tile may not cross pages): fp32 FMA
  ProjectParams p{ls.k, ls.kimp, ls.wk, c.n_kv_heads, c.max_len, start, count, ls.kl, c.kimp_bf16};
  dim3 grid((count + kProjRows - 1) / kProjRows, c.n_kv_heads, c.batch);
#define TB_PROJ_CASE(T, DV, DI) \
  if (c.head_dim == DV && c.d_imp == DI) project_fma_kernel<T, DV, DI><<<grid, 256, 0, st>>>(p); else
  if (c.kv_dtype == TB_BF16) {
    TB_PROJ_CASE(__nv_bfloat16, 128, 32) TB_PROJ_CASE(__nv_bfloat16, 128, 16) TB_PROJ_CASE(__nv_bfloat16, 64, 32)
    TB_PROJ_CASE(__nv_bfloat16, 64, 16) return TB_ERR_UNSUPPORTED;
  } else {
    TB_PROJ_CASE(float, 128, 32) TB_PROJ_CASE(float, 128, 16) TB_PROJ_CASE(float, 64, 32)
    TB_PROJ_CASE(float, 64, 16) return TB_ERR_UNSUPPORTED;
  }
#undef TB_PROJ_CASE
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_project_kimp_layers(tb_ctx* ctx, int first_layer, int n_layers, int start, int count,
                                        void* stream) {
  if (!ctx || n_layers < 1 || first_layer < 0 || (long long)first_layer + n_layers > ctx->cfg.n_layers)
    return TB_ERR_INVALID_ARG;
  const tb_config& c = ctx->cfg;
  if (start < 0 || count < 0 || (long long)start + count > c.max_len) return TB_ERR_CAPACITY;
  bool tc = c.kv_dtype == TB_BF16;
  for (int l = first_layer; l < first_layer + n_layers; ++l) {
    const tb_status s = check_layer(ctx, l);
    if (s != TB_OK) return s;
    tc = tc && ctx->layers[l].kl.page_table == nullptr;
  }
  if (count == 0) return TB_OK;
  if (!tc) {  // fp32 or paged caches: the FMA projection, layer by layer
    for (int l = first_layer; l < first_layer + n_layers; ++l) {
      const tb_status s = tb_project_kimp(ctx, l, start, count, stream);
      if (s != TB_OK) return s;
    }
    return TB_OK;
  }
  return launch_project_tc(ctx, first_layer, n_layers, start, count, static_cast<cudaStream_t>(stream));
}

TB_API tb_status tb_score(tb_ctx* ctx, int layer, const void* q_imp_producer, float* scores, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!q_imp_producer || !scores) return TB_ERR_INVALID_ARG;
  if (!aligned16(scores)) return TB_ERR_SHAPE;
  return launch_score(ctx, layer, q_imp_producer, scores, nullptr, static_cast<cudaStream_t>(stream));
}

TB_API tb_status tb_select(tb_ctx* ctx, int layer, const float* scores, int rows_per_seq, int32_t* idx,
                           int idx_cap, int32_t* count, uint32_t* mask, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  const tb_config& c = ctx->cfg;
  if (!scores || (!idx && !count && !mask)) return TB_ERR_INVALID_ARG;
  if (rows_per_seq != c.n_q_heads && rows_per_seq != c.n_kv_heads && rows_per_seq != 1) return TB_ERR_SHAPE;
  if (!aligned16(scores)) return TB_ERR_SHAPE;
  if (idx) {
    const LayerState& ls = ctx->layers[layer];
    for (int b = 0; b < c.batch; ++b) {
      const long long L = ls.lens[b];
      const long long nc = std::max(0LL, L - c.window - c.sink);
      const long long k = std::min((long long)c.keep_pct * L / 100, nc);
      const long long sink_n = std::min<long long>(c.sink, L);
      const long long win_lo = std::max(L - c.window, sink_n);
      if (sink_n + (L - win_lo) + k > idx_cap) return TB_ERR_SHAPE;
    }
  }
  return launch_select(ctx, layer, scores, false, rows_per_seq, idx, idx_cap, count, mask,
                       static_cast<cudaStream_t>(stream));
}

TB_API tb_status tb_sparse_attn(tb_ctx* ctx, int layer, const void* q, const uint32_t* mask, int mask_mode,
                                void* out, float* lse, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!q || !out) return TB_ERR_INVALID_ARG;
  if (mask_mode != TB_MASK_PER_HEAD && mask_mode != TB_MASK_SHARED && mask_mode != TB_MASK_DENSE &&
      mask_mode != TB_MASK_GROUP)
    return TB_ERR_INVALID_ARG;
  if (mask_mode != TB_MASK_DENSE && !mask) return TB_ERR_INVALID_ARG;
  if (!aligned16(q)) return TB_ERR_SHAPE;
  return launch_attn(ctx, layer, q, mask, mask_mode, out, lse, static_cast<cudaStream_t>(stream));
}

TB_API tb_status tb_sparse_attn_idx(tb_ctx* ctx, int layer, const void* q, const int32_t* idx, int idx_cap,
                                    const int32_t* count, void* out, float* lse, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!q || !idx || !count || !out || idx_cap < 1) return TB_ERR_INVALID_ARG;
  if (!aligned16(q)) return TB_ERR_SHAPE;
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  IndexMaskParams p{};
  p.idx = idx;
  p.count = count;
  p.mask = ctx->mask;
  p.status = ctx->status;
  p.Hq = c.n_q_heads;
  p.idx_cap = idx_cap;
  p.mask_words = c.max_len / 32;
  for (int b = 0; b < c.batch; ++b) p.lens[b] = ls.lens[b];
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  launch_pdl(index_mask_kernel, dim3(c.n_q_heads, c.batch), dim3(kIdxMaskThreads), 0, st, p);
  ++ctx->launches;
  s = cuda_status(cudaGetLastError());
  if (s != TB_OK) return s;
  return launch_attn(ctx, layer, q, ctx->mask, TB_MASK_PER_HEAD, out, lse, st);
}

// Amortised selection: per-row reuse decisions of this step (see reuse.cuh).
static tb_status launch_reuse_decide(tb_ctx* ctx, int layer, const void* q_imp, cudaStream_t st) {
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  ReuseParams p{};
  p.q_imp = q_imp;
  p.sc_q = ls.sc_q;
  p.sc_len = ls.sc_len;
  p.reuse = ctx->reuse;
  p.G = c.producer_freq;
  p.slot = ((layer - 1) % c.producer_freq + c.producer_freq) % c.producer_freq;
  p.Hq = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.rows_per_seq = sel_rows(c);
  p.nrows_total = c.batch * p.rows_per_seq;
  p.tau = ctx->reuse_tau;
  p.interval = ctx->reuse_interval;
  p.keep_pct = c.keep_pct;
  p.sink = c.sink;
  p.window = c.window;
  for (int b = 0; b < c.batch; ++b) p.lens[b] = ls.lens[b];
  const dim3 grid((p.nrows_total + 7) / 8);
  if (c.kv_dtype == TB_BF16) {
    if (c.d_imp == 32) launch_pdl(reuse_decide_kernel<__nv_bfloat16, 32>, grid, dim3(256), 0, st, p);
    else launch_pdl(reuse_decide_kernel<__nv_bfloat16, 16>, grid, dim3(256), 0, st, p);
  } else {
    if (c.d_imp == 32) launch_pdl(reuse_decide_kernel<float, 32>, grid, dim3(256), 0, st, p);
    else launch_pdl(reuse_decide_kernel<float, 16>, grid, dim3(256), 0, st, p);
  }
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_decode_step(tb_ctx* ctx, int layer, const void* k_new, const void* v_new, const void* q,
                                const void* q_imp_producer, void* out, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  const tb_config& c = ctx->cfg;
  if (!k_new || !v_new || !q || !out) return TB_ERR_INVALID_ARG;
  const bool dense = ((c.dense_layer_mask >> layer) & 1ull) || c.keep_pct >= 100;
  if (!dense && c.variant != TB_SOFTVOTE && !q_imp_producer) return TB_ERR_INVALID_ARG;
  if (!aligned16(q)) return TB_ERR_SHAPE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  trace_point(ctx, 0, st);
  s = tb_append_kv(ctx, layer, k_new, v_new, stream);
  if (s != TB_OK) return s;
  trace_point(ctx, 1, st);
  if (dense) {
    trace_point(ctx, 2, st);
    trace_point(ctx, 3, st);
    return launch_attn(ctx, layer, q, nullptr, TB_MASK_DENSE, out, nullptr, st);
  }
  if (c.variant == TB_BUTLER || c.variant == TB_BUTLER_GROUP) {
    const bool grouped = c.variant == TB_BUTLER_GROUP;
    const LayerState& ls = ctx->layers[layer];
    const bool cached = ls.sc_q != nullptr && ctx->reuse_interval > 0;
    if (cached) {
      s = launch_reuse_decide(ctx, layer, q_imp_producer, st);
      if (s != TB_OK) return s;
    }
    s = launch_score(ctx, layer, q_imp_producer, ctx->scores, ctx->hist, st, cached ? ctx->reuse : nullptr);
    if (s != TB_OK) return s;
    trace_point(ctx, 2, st);
    s = launch_select(ctx, layer, ctx->scores, true, grouped ? c.n_kv_heads : c.n_q_heads, nullptr, 0, nullptr,
                      ctx->mask, st, cached, true);
    if (s != TB_OK) return s;
    trace_point(ctx, 3, st);
    return launch_attn(ctx, layer, q, ctx->mask, grouped ? TB_MASK_GROUP : TB_MASK_PER_HEAD, out, nullptr, st);
  }
  // soft voting: votes over the full K (the appended row included), one shared set
  prepare_hist(ctx, st);
  s = launch_softvote(ctx, layer, q, ctx->votes, ctx->hist, st);
  if (s != TB_OK) return s;
  trace_point(ctx, 2, st);
  s = launch_select(ctx, layer, ctx->votes, true, 1, nullptr, 0, nullptr, ctx->mask, st, false, true);
  if (s != TB_OK) return s;
  trace_point(ctx, 3, st);
  return launch_attn(ctx, layer, q, ctx->mask, TB_MASK_SHARED, out, nullptr, st);
}

TB_API tb_status tb_select_prefill(tb_ctx* ctx, int layer, const void* q_imp_rows, int row0, int nrows,
                                   uint32_t* row_masks, int words_per_row, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  if (!q_imp_rows || !row_masks) return TB_ERR_INVALID_ARG;
  if (row0 < 0 || nrows < 0) return TB_ERR_INVALID_ARG;
  if (nrows == 0) return TB_OK;
  const long long need = (long long)row0 + nrows;
  if (need > c.max_len) return TB_ERR_CAPACITY;
  if (words_per_row < (need + 31) / 32) return TB_ERR_SHAPE;
  for (int b = 0; b < c.batch; ++b)
    if (ls.lens[b] < need) return TB_ERR_STATE;  // K_imp rows of the prefix must exist
  if (need > kPfMaxPrefix) return TB_ERR_UNSUPPORTED;  // the one-row method keeps row scores in shared memory
  const size_t smem = (size_t)need * 4;
  PrefillParams p{};
  p.q_imp = q_imp_rows;
  p.kimp = ls.kimp;
  p.masks = row_masks;
  p.status = ctx->status;
  p.G = c.producer_freq;
  p.slot = ((layer - 1) % c.producer_freq + c.producer_freq) % c.producer_freq;
  p.Hq = c.n_q_heads;
  p.Hkv = c.n_kv_heads;
  p.max_len = c.max_len;
  p.row0 = row0;
  p.nrows = nrows;
  p.words_per_row = words_per_row;
  p.keep_pct = c.keep_pct;
  p.sink = c.sink;
  p.window = c.window;
  // rows the blocked kernel hands over to the one-row method are flagged in
  // the score workspace (B * Hq * nrows words <= B * Hq * max_len floats)
  p.redo = reinterpret_cast<uint32_t*>(ctx->scores);
  dim3 grid((nrows + kPfRows - 1) / kPfRows, c.n_q_heads, c.batch);
  dim3 rgrid((unsigned)std::min<long long>(ctx->num_sms, (long long)c.n_q_heads * nrows), c.batch);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
#define TB_PF_CASE(T, KT, DI)                                                           \
  if (c.d_imp == DI) {                                                                  \
    auto kb = prefill_rows_kernel<T, KT, DI>;                                           \
    if (cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, kPfSmem) != cudaSuccess) \
      return TB_ERR_CUDA;                                                                            \
    kb<<<grid, kPfThreads, kPfSmem, st>>>(p);                                           \
    auto kr = prefill_redo_kernel<T, KT, DI>;                                           \
    if (cudaFuncSetAttribute(kr, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) \
      return TB_ERR_CUDA;                                                                            \
    kr<<<rgrid, kSelThreads, smem, st>>>(p);                                            \
    ctx->launches += 2;                                                                 \
  } else
  if (c.kv_dtype == TB_BF16 && c.kimp_bf16) {
    TB_PF_CASE(__nv_bfloat16, __nv_bfloat16, 32) TB_PF_CASE(__nv_bfloat16, __nv_bfloat16, 16) return TB_ERR_UNSUPPORTED;
  } else if (c.kv_dtype == TB_BF16) {
    TB_PF_CASE(__nv_bfloat16, float, 32) TB_PF_CASE(__nv_bfloat16, float, 16) return TB_ERR_UNSUPPORTED;
  } else {
    TB_PF_CASE(float, float, 32) TB_PF_CASE(float, float, 16) return TB_ERR_UNSUPPORTED;
  }
#undef TB_PF_CASE
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_softvote_scores(tb_ctx* ctx, int layer, const void* q, float* votes, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!q || !votes) return TB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(votes)) return TB_ERR_SHAPE;
  return launch_softvote(ctx, layer, q, votes, nullptr, static_cast<cudaStream_t>(stream));
}

TB_API tb_status tb_trace_events(tb_ctx* ctx, void* const* events, int n_events) {
  if (!ctx) return TB_ERR_INVALID_ARG;
  if (!events) {
    ctx->tracing = false;
    return TB_OK;
  }
  if (n_events != 6) return TB_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i) {
    if (!events[i]) return TB_ERR_INVALID_ARG;
    ctx->trace[i] = static_cast<cudaEvent_t>(events[i]);
  }
  ctx->tracing = true;
  return TB_OK;
}

TB_API tb_status tb_launch_count(const tb_ctx* ctx, uint64_t* count) {
  if (!ctx || !count) return TB_ERR_INVALID_ARG;
  *count = ctx->launches;
  return TB_OK;
}

// Failure-detection self-test of the library's bounded mbarrier wait
// (mbar_wait, as used by the pipelined kernels): one mbarrier that expects
// one arrival.  With `arrive`, thread 0 arrives and the wait
// completes; otherwise nothing arrives, the wait gives up after `cycles` SM
// cycles and TB_DEV_ERR_TIMEOUT is recorded.  The CTA then exits normally.
static __global__ void wait_selftest_kernel(uint32_t* status, long long cycles, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    mbar_fence_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive_cta(&bar);
    if (!mbar_wait(&bar, 0, cycles)) atomicOr(status, TB_DEV_ERR_TIMEOUT);
  }
}

TB_API tb_status tb_selftest_bounded_wait(tb_ctx* ctx, long long cycles, int arrive, void* stream) {
  if (!ctx) return TB_ERR_INVALID_ARG;
  if (cycles < 1 || cycles > 20000000000LL) return TB_ERR_INVALID_ARG;  // at most about ten seconds
  wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(ctx->status, cycles, arrive ? 1 : 0);
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_check_status(tb_ctx* ctx, uint32_t* flags) {
  if (!ctx) return TB_ERR_INVALID_ARG;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ctx->status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return TB_ERR_CUDA;
  if (v && cudaMemset(ctx->status, 0, sizeof(v)) != cudaSuccess) return TB_ERR_CUDA;
  if (flags) *flags = v;
  return v ? TB_ERR_DEVICE_STATUS : TB_OK;
}

TB_API const char* tb_status_string(tb_status s) {
  switch (s) {
    case TB_OK: return "ok";
    case TB_ERR_INVALID_ARG: return "invalid argument";
    case TB_ERR_SHAPE: return "unsupported shape or alignment";
    case TB_ERR_CAPACITY: return "sequence length exceeds cache capacity";
    case TB_ERR_WORKSPACE: return "workspace missing or too small";
    case TB_ERR_CUDA: return "CUDA error";
    case TB_ERR_DEVICE_STATUS: return "a kernel reported an error";
    case TB_ERR_UNSUPPORTED: return "not supported by this build";
    case TB_ERR_STATE: return "layer not bound";
  }
  return "unknown status";
}

TB_API void tb_destroy(tb_ctx* ctx) { delete ctx; }

}  // extern "C"

// ------------------------------------------------------------------ sequence sharding
static tb_status shard_params(const tb_ctx* ctx, int layer, ShardParams* p) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  const tb_config& c = ctx->cfg;
  const LayerState& ls = ctx->layers[layer];
  if (c.variant == TB_SOFTVOTE) return TB_ERR_UNSUPPORTED;
  if (!ls.shard_on) return TB_ERR_STATE;
  *p = ShardParams{};
  p->status = ctx->status;
  p->rows = sel_rows(c);
  p->total_rows = c.batch * p->rows;
  p->max_len = c.max_len;
  p->keep_pct = c.keep_pct;
  p->sink = c.sink;
  p->window = c.window;
  p->t0 = ls.shard_t0;
  for (int b = 0; b < c.batch; ++b) {
    p->nloc[b] = ls.lens[b];
    p->glen[b] = ls.glen[b];
  }
  return TB_OK;
}

TB_API tb_status tb_shard_set(tb_ctx* ctx, int layer, int t0, const int32_t* global_lens) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!global_lens || t0 < 0) return TB_ERR_INVALID_ARG;
  const tb_config& c = ctx->cfg;
  if (c.variant == TB_SOFTVOTE) return TB_ERR_UNSUPPORTED;
  LayerState& ls = ctx->layers[layer];
  for (int b = 0; b < c.batch; ++b)
    if ((long long)t0 + ls.lens[b] > global_lens[b] || global_lens[b] < 0) return TB_ERR_STATE;
  ls.shard_on = true;
  ls.shard_t0 = t0;
  for (int b = 0; b < c.batch; ++b) ls.glen[b] = global_lens[b];
  return TB_OK;
}

static unsigned shard_chunks(const tb_ctx* ctx, const ShardParams& p, int tok) {
  int m = 1;
  for (int b = 0; b < ctx->cfg.batch; ++b) m = std::max(m, p.nloc[b]);
  return (unsigned)((m + tok - 1) / tok);
}

TB_API tb_status tb_shard_hist(tb_ctx* ctx, int layer, const float* scores, int pass, const uint32_t* state,
                               uint32_t* hist, void* stream) {
  ShardParams p;
  tb_status s = shard_params(ctx, layer, &p);
  if (s != TB_OK) return s;
  if (!scores || !hist || (pass > 0 && !state) || pass < 0 || pass > 2) return TB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  p.scores = scores;
  p.state = reinterpret_cast<uint4*>(const_cast<uint32_t*>(state));
  p.hist = hist;
  p.pass = pass;
  const size_t n = (size_t)p.total_rows * kHistBins;
  launch_pdl(zero_u32_kernel, dim3((unsigned)std::min<size_t>((n + 255) / 256, 1024)), dim3(256), 0, st, hist, n);
  launch_pdl(shard_hist_kernel, dim3(shard_chunks(ctx, p, kShardHistTok), p.total_rows), dim3(kShardThreads), 0, st,
             p);
  ctx->launches += 2;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_shard_pick(tb_ctx* ctx, int layer, int pass, const uint32_t* hist, int n_ranks, int rank,
                               uint32_t* state, void* stream) {
  ShardParams p;
  tb_status s = shard_params(ctx, layer, &p);
  if (s != TB_OK) return s;
  if (!hist || !state || pass < 0 || pass > 2) return TB_ERR_INVALID_ARG;
  if (n_ranks < 1 || rank < 0 || rank >= n_ranks || (pass < 2 && n_ranks != 1)) return TB_ERR_INVALID_ARG;
  p.hist_in = hist;
  p.state = reinterpret_cast<uint4*>(state);
  p.pass = pass;
  p.n_ranks = n_ranks;
  p.rank = rank;
  launch_pdl(shard_pick_kernel, dim3((unsigned)p.total_rows), dim3(kShardThreads), 0,
             static_cast<cudaStream_t>(stream), p);
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_shard_mask(tb_ctx* ctx, int layer, const float* scores, const uint32_t* state, uint32_t* mask,
                               void* stream) {
  ShardParams p;
  tb_status s = shard_params(ctx, layer, &p);
  if (s != TB_OK) return s;
  if (!scores || !state || !mask) return TB_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  p.scores = scores;
  p.state = reinterpret_cast<uint4*>(const_cast<uint32_t*>(state));
  p.mask = mask;
  launch_pdl(shard_mask_kernel, dim3(shard_chunks(ctx, p, kShardMaskTok), p.total_rows), dim3(kShardThreads), 0, st,
             p);
  launch_pdl(shard_ties_kernel, dim3((unsigned)p.total_rows), dim3(kShardThreads), 0, st, p);
  ctx->launches += 2;
  return cuda_status(cudaGetLastError());
}

TB_API tb_status tb_sparse_attn_partial(tb_ctx* ctx, int layer, const void* q, const uint32_t* mask, int mask_mode,
                                        float* part, void* stream) {
  tb_status s = check_layer(ctx, layer);
  if (s != TB_OK) return s;
  if (!q || !part) return TB_ERR_INVALID_ARG;
  if (mask_mode != TB_MASK_PER_HEAD && mask_mode != TB_MASK_SHARED && mask_mode != TB_MASK_GROUP &&
      mask_mode != TB_MASK_DENSE)
    return TB_ERR_INVALID_ARG;
  if (mask_mode != TB_MASK_DENSE && !mask) return TB_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(part)) return TB_ERR_SHAPE;
  const tb_config& c = ctx->cfg;
  float* lse = part + (size_t)c.batch * c.n_q_heads * c.head_dim;
  return launch_attn(ctx, layer, q, mask, mask_mode, part, lse, static_cast<cudaStream_t>(stream), true);
}

TB_API tb_status tb_merge_partials(tb_ctx* ctx, const float* parts, int n_parts, void* out, float* lse,
                                   void* stream) {
  if (!ctx || !parts || !out || n_parts < 1) return TB_ERR_INVALID_ARG;
  const tb_config& c = ctx->cfg;
  MergeParams p{};
  p.parts = parts;
  p.rows = c.batch * c.n_q_heads;
  p.part_stride = (size_t)p.rows * (c.head_dim + 1);
  p.out = out;
  p.lse = lse;
  p.n_parts = n_parts;
  const dim3 grid((unsigned)((p.rows + 3) / 4));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (c.kv_dtype == TB_BF16) {
    if (c.head_dim == 128) launch_pdl(merge_partials_kernel<__nv_bfloat16, 128>, grid, dim3(128), 0, st, p);
    else launch_pdl(merge_partials_kernel<__nv_bfloat16, 64>, grid, dim3(128), 0, st, p);
  } else {
    if (c.head_dim == 128) launch_pdl(merge_partials_kernel<float, 128>, grid, dim3(128), 0, st, p);
    else launch_pdl(merge_partials_kernel<float, 64>, grid, dim3(128), 0, st, p);
  }
  ++ctx->launches;
  return cuda_status(cudaGetLastError());
}
