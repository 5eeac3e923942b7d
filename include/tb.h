/*
 * tb.h — C ABI of the TokenButler decode-step hot path on B200 (sm_100a).
 *
 * Each decode step of a consumer layer l:
 *   1. appends the new token's key/value and its importance key
 *      K_imp = K . W_K  (model card "Meta-Llama-3.1-8B-Instruct-Butler",
 *      section "Method": learned projection of the real post-RoPE keys);
 *   2. scores every cached token with the importance query that the layer's
 *      producer (layer G*floor(l/G)) emitted in slot (l - 1) mod G
 *      (same section: producers at layers 0, G, 2G, ...);
 *   3. keeps, per query head, the top-k tokens under a fixed budget plus a
 *      sink prefix and a recent local window (same section; budget policy
 *      fixed_<N>pc, min_sparse_index and sliding_window in section
 *      "Memory requirements"; layer 0 dense);
 *   4. runs exact attention over only the kept tokens of the untouched full
 *      KV cache (model card introduction; TokenButler abstract: "fixed
 *      budget while preserving the full KV cache").
 * The soft-voting variant (TokenSelect README, "Per-head Soft Voting
 * Mechanism") replaces 2-3 by one ranking shared by all heads: per-head
 * softmax of q . K / sqrt(D), summed over the heads.
 *
 * Conventions
 *   - Ownership: the caller owns every buffer (caches, W_K, queries, outputs,
 *     workspace).  The library never allocates or frees device memory; a
 *     tb_ctx is a small host object that records pointers and lengths.
 *   - Pointers named *_cache, q*, k_new, v_new, out, scores, idx, count, mask,
 *     lse and the workspace are DEVICE pointers; *_host arguments are host
 *     pointers.  `stream` is a cudaStream_t (NULL = legacy default stream).
 *   - All compute calls are asynchronous on `stream`.  Argument and shape
 *     errors are detected on the host and returned synchronously before
 *     anything is launched; TB_ERR_CUDA reports a launch error.  Errors seen
 *     by a kernel set bits of a device status word, read by tb_check_status()
 *     after a synchronisation.  Nothing aborts, traps or throws.
 *   - Layouts are dense and row-major (last index fastest):
 *       K cache, V cache   [B][Hkv][max_len][D]   kv_dtype
 *       K_imp cache        [B][Hkv][max_len/256][d'][256]  fp32, or bf16 when
 *                          cfg.kimp_bf16 = 1: tiles of 256 tokens, each
 *                          contiguous and dimension-major (element (b, g, t, j)
 *                          at tile t/256, row j, column t%256)
 *       W_K                [D][d']                kv_dtype
 *       q_imp (producer)   [(B*Hq)][G][n][d']     kv_dtype  (model card: (B.H) x G x L x d')
 *       q, out             [B][Hq][D]             kv_dtype
 *       k_new, v_new       [B][Hkv][D]            kv_dtype
 *       scores             [B][Hq][max_len]       fp32
 *       mask (per head)    [B][Hq][max_len/32]    uint32, bit t%32 of word t/32
 *       mask (shared)      [B][max_len/32]        uint32  (soft voting)
 *       idx                [B][Hq][idx_cap]       int32, ascending
 *       count, lse         [B][Hq]                int32 / fp32
 *     Every device pointer must be 16-byte aligned; max_len must be a
 *     multiple of 256.
 *   - Query head h reads KV head h / (Hq / Hkv).
 *   - Sequence b of layer l holds len[l][b] tokens (tb_set_seq_lens /
 *     tb_append_kv); the decode query sits at position len - 1.
 *   - Selection (per query head, per sequence, L = len):
 *       k = floor(keep_pct * L / 100); candidates C = [sink, L - window);
 *       Sel = [0, min(sink, L)) U top_min(k,|C|)(C) U [max(L - window, 0), L)
 *     top-k orders by (score descending, index ascending); -0.0 == +0.0;
 *     NaN scores are outside the contract.
 *   - A tb_ctx is not re-entrant across concurrent streams.
 */
#ifndef TB_H
#define TB_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define TB_API __attribute__((visibility("default")))
#else
#define TB_API
#endif

typedef enum {
  TB_OK = 0,
  TB_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, negative size        */
  TB_ERR_SHAPE = 2,         /* shape/alignment not supported                */
  TB_ERR_CAPACITY = 3,      /* a sequence would exceed max_len              */
  TB_ERR_WORKSPACE = 4,     /* workspace missing or too small               */
  TB_ERR_CUDA = 5,          /* CUDA runtime / launch error                  */
  TB_ERR_DEVICE_STATUS = 6, /* a kernel flagged an error (tb_check_status)  */
  TB_ERR_UNSUPPORTED = 7,   /* valid request this build does not implement  */
  TB_ERR_STATE = 8          /* layer not bound / lengths not set            */
} tb_status;

typedef enum { TB_BF16 = 0, TB_F32 = 1 } tb_dtype;
/* TB_BUTLER: one selection per query head (model card "Method").
 * TB_SOFTVOTE: one selection per sequence from soft votes (TokenSelect README).
 * TB_BUTLER_GROUP: one selection per KV group: the importance scores of the
 *   group's Hq/Hkv query heads are summed (fp32, in head order) and the group
 *   selects once.  This is a GQA-aware option, not a reading of the pages:
 *   the pages select per head.  Every K/V row the group reads is then used by
 *   all of its heads, so the attention reads far fewer rows. */
typedef enum { TB_BUTLER = 0, TB_SOFTVOTE = 1, TB_BUTLER_GROUP = 2 } tb_variant;
typedef enum { TB_MASK_PER_HEAD = 0, TB_MASK_SHARED = 1, TB_MASK_DENSE = 2, TB_MASK_GROUP = 3 } tb_mask_mode;

/* device status word bits (tb_check_status) */
#define TB_DEV_ERR_INDEX 0x1u     /* a gathered index was outside [0, len)    */
#define TB_DEV_ERR_COUNT 0x2u     /* a selected-set size differed from k      */
#define TB_DEV_ERR_TIMEOUT 0x4u   /* a bounded wait gave up                   */

#define TB_MAX_BATCH 128
#define TB_MAX_LAYERS 64

typedef struct tb_config {
  int n_layers;              /* decoder layers, 1..TB_MAX_LAYERS                          */
  int batch;                 /* B, 1..TB_MAX_BATCH                                        */
  int n_q_heads;             /* Hq                                                        */
  int n_kv_heads;            /* Hkv; Hq % Hkv == 0, Hq/Hkv in {1,2,4,8}                   */
  int head_dim;              /* D in {64, 128}                                            */
  int d_imp;                 /* d' in {16, 32}                                            */
  int producer_freq;         /* G >= 1 (model card "Method")                              */
  int max_len;               /* cache capacity per sequence, multiple of 256             */
  int kv_dtype;              /* tb_dtype of K, V, W_K, q, q_imp, out                       */
  int keep_pct;              /* P: 100 - N of the fixed_<N>pc policy, 0..100              */
  int sink;                  /* min_sparse_index: always-kept prefix length               */
  int window;                /* sliding_window: always-kept recent tokens                 */
  uint64_t dense_layer_mask; /* bit l set: layer l attends densely (layer 0 by default)   */
  int variant;               /* tb_variant                                                */
  int kimp_bf16;             /* 0: fp32 K_imp cache (default); 1: bf16 K_imp cache, every
                                K_imp value computed in fp32 and rounded to nearest even
                                (halves the score stream; kv_dtype TB_BF16 only, else
                                TB_ERR_UNSUPPORTED).  Option beyond the pages, which do not
                                state the cache's precision                               */
} tb_config;

typedef struct tb_ctx tb_ctx;

/* Bytes of device workspace tb_init needs for `cfg` (host-only, no CUDA call). */
TB_API tb_status tb_workspace_size(const tb_config* cfg, size_t* bytes);

/* Validate `cfg` and create a context on the current CUDA device.
 * `workspace`: caller-owned device buffer of >= tb_workspace_size bytes,
 * 256-byte aligned, alive until tb_destroy.  Its contents need no
 * initialisation.  *out receives a host object freed by tb_destroy. */
TB_API tb_status tb_init(const tb_config* cfg, void* workspace, size_t ws_bytes, tb_ctx** out);

/* Register layer `layer`'s caller-owned caches and W_K (device pointers,
 * layouts above).  All lengths of the layer start at 0. */
TB_API tb_status tb_bind_layer(tb_ctx* ctx, int layer, void* k_cache, void* v_cache, void* kimp_cache,
                               const void* w_k);

/* Paged K/V caches (serving layouts: the attention's page-table gather).
 * Register layer `layer` with K and V page pools [num_pages][Hkv][page_size][D]
 * (kv_dtype) and a device page table `page_table` [B][max_pages] int32: token
 * t of sequence b, KV head g, is row t % page_size of page
 * page_table[b][t / page_size].  page_size: a power of two >= 16;
 * max_pages * page_size >= max_len; num_pages * Hkv * page_size < 2^31.  The
 * table is read by the kernels, so the caller may remap pages between calls
 * (stream-ordered).  K_imp stays a dense per-sequence cache as above.  Every
 * call works on paged layers; the K_imp projection of paged bf16 caches uses
 * fp32 FMA instead of the tensor cores (a TMA tile may not cross pages).
 * Lengths start at 0. */
TB_API tb_status tb_bind_layer_paged(tb_ctx* ctx, int layer, void* k_pool, void* v_pool, int num_pages,
                                     const int32_t* page_table, int page_size, int max_pages, void* kimp_cache,
                                     const void* w_k);

/* Set / read the per-sequence lengths of a layer (host arrays of `batch`
 * int32).  Used after the caller filled the caches by a prefill. */
TB_API tb_status tb_set_seq_lens(tb_ctx* ctx, int layer, const int32_t* lens_host);
TB_API tb_status tb_get_seq_lens(const tb_ctx* ctx, int layer, int32_t* lens_host);

/* Runtime budget setters: the model card's set_token_sparsity() /
 * min_sparse_index / sliding_window knobs ("Memory requirements"). */
TB_API tb_status tb_set_budget(tb_ctx* ctx, int keep_pct, int sink, int window);

/* a1 — model card "Method", K_imp = K . W_K, decode side.  Writes k_new and
 * v_new ([B][Hkv][D]) at position len[b] of every sequence, computes that
 * row's K_imp in fp32 (stored in the cache's type), then increments len[b] (host-side bookkeeping at
 * enqueue time).  TB_ERR_CAPACITY if a sequence is full. */
TB_API tb_status tb_append_kv(tb_ctx* ctx, int layer, const void* k_new, const void* v_new, void* stream);

/* a1' — model card "Method", K_imp = K . W_K, prefill side: computes K_imp
 * rows [start, start + count) of every (b, KV head) from the cached K.
 * bf16 caches run on the tensor cores (tcgen05, fp32 accumulation); fp32
 * caches use fp32 FMA (no TF32).  A bf16 K_imp cache receives each fp32
 * result rounded to nearest even. */
TB_API tb_status tb_project_kimp(tb_ctx* ctx, int layer, int start, int count, void* stream);

/* a1' for layers [first_layer, first_layer + n_layers) at once (same rows
 * [start, start + count) of each): with dense bf16 caches one persistent
 * tensor-core launch covers every layer's tiles (a prefill of all layers
 * streams K at the HBM rate instead of paying one short launch per layer);
 * fp32 or paged caches run tb_project_kimp layer by layer.  Each result
 * equals tb_project_kimp's bit for bit. */
TB_API tb_status tb_project_kimp_layers(tb_ctx* ctx, int first_layer, int n_layers, int start, int count,
                                        void* stream);

/* a2 + a3 — model card "Method": scores[b][h][t] = q_hat[b][h] . K_imp[b][g(h)][t]
 * for t < len[b], with q_hat[b][h] = q_imp_producer[b*Hq + h][(layer-1) mod G][0][:]
 * (fp32 FMA on the stored K_imp values, no scale).  `q_imp_producer`: [(B*Hq)][G][1][d'] of producer
 * G*floor(layer/G).  Entries t >= len[b] are left untouched.  With
 * TB_BUTLER_GROUP the rows are per KV group instead ([B][Hkv][max_len]):
 * scores[b][g][t] = sum over the group's heads, in head order, of the fp32
 * per-head scores. */
TB_API tb_status tb_score(tb_ctx* ctx, int layer, const void* q_imp_producer, float* scores, void* stream);

/* a4 + a5 — model card "Method" / "Memory requirements": per row of `scores`
 * ([B][rows_per_seq][max_len]; rows_per_seq is Hq for per-head sets, Hkv for
 * per-group sets, 1 for a shared ranking), selects Sel as in the header
 * comment, with the budget of the context.  Outputs (each may be NULL, not all):
 *   idx   [B][rows][idx_cap] ascending indices (TB_ERR_SHAPE if idx_cap is
 *         smaller than the largest selected set),
 *   count [B][rows] selected-set sizes,
 *   mask  [B][rows][max_len/32] bitmask; words past ceil(len/32) untouched.
 * Bit-exact: the choice depends only on the fp32 score values. */
TB_API tb_status tb_select(tb_ctx* ctx, int layer, const float* scores, int rows_per_seq, int32_t* idx,
                           int idx_cap, int32_t* count, uint32_t* mask, void* stream);

/* a6 — exact attention over a selected set of the untouched cache:
 * out[b][h] = sum_{t in Sel} softmax_t(q[b][h] . K[b][g(h)][t] / sqrt(D)) V[b][g(h)][t]
 * (fp32 accumulation).  `mask_mode`: TB_MASK_PER_HEAD (mask [B][Hq][max_len/32]),
 * TB_MASK_GROUP (mask [B][Hkv][max_len/32], one set per KV group),
 * TB_MASK_SHARED (mask [B][max_len/32], one set per sequence) or
 * TB_MASK_DENSE (mask NULL: every token t < len, the layer-0 / 100 % path).
 * `lse` (optional, [B][Hq] fp32): natural log of the softmax denominator;
 * an empty set gives out = 0 and lse = -inf.  Split-K over token chunks with
 * an fp32 log-sum-exp merge; each K/V row is read once per KV head. */
TB_API tb_status tb_sparse_attn(tb_ctx* ctx, int layer, const void* q, const uint32_t* mask, int mask_mode,
                                void* out, float* lse, void* stream);

/* a6 with the selected sets as index lists, the shape tb_select writes:
 * idx [B][Hq][idx_cap] int32 token indices (each listed once; any order),
 * count [B][Hq] int32 (device).  The lists are turned into per-head
 * bitmasks in the context's workspace (what tb_copy_step_masks copies is
 * then these sets), then tb_sparse_attn runs in TB_MASK_PER_HEAD mode: the
 * same result as tb_sparse_attn on the equivalent mask.  An index outside
 * [0, len) is skipped, a count outside [0, idx_cap] is clamped, and either
 * sets TB_DEV_ERR_INDEX. */
TB_API tb_status tb_sparse_attn_idx(tb_ctx* ctx, int layer, const void* q, const int32_t* idx, int idx_cap,
                                    const int32_t* count, void* out, float* lse, void* stream);

/* a1..a6 for one layer: append, then (dense layer or 100 % budget) dense
 * attention, else score, select and sparse attention (TB_BUTLER per head,
 * TB_BUTLER_GROUP per KV group) or soft voting with a shared set
 * (TB_SOFTVOTE; q_imp_producer unused).  Uses the workspace for scores,
 * masks and split partials.  The workspace scores are dropped from L2
 * without a write-back once the selection has read them (their contents are
 * undefined after the call; the masks are kept). */
TB_API tb_status tb_decode_step(tb_ctx* ctx, int layer, const void* k_new, const void* v_new, const void* q,
                                const void* q_imp_producer, void* out, void* stream);

/* a7 — prefill rows of a consumer layer: for positions p in
 * [row0, row0 + nrows) and every (b, h), scores the causal prefix
 * s_p[t] = q_hat[b][h][p] . K_imp[b][g(h)][t], t <= p, and selects with
 * L -> p + 1.  `q_imp_rows`: [(B*Hq)][G][nrows][d'] (positions row0..), slot
 * (layer-1) mod G.  `row_masks`: [B][Hq][nrows][words_per_row] uint32 with
 * words_per_row >= ceil((row0 + nrows)/32); every word is written.
 * Requires len[b] >= row0 + nrows (K_imp rows present) and
 * row0 + nrows <= 51200 (a row's fp32 scores fit 200 KB of shared memory for
 * the massive-ties method), else TB_ERR_UNSUPPORTED.  Rows are scored in
 * blocks of 16 on the tensor cores (TF32 with an fp32 K_imp split into a TF32 head
 * and its remainder, fp32 accumulation: about 1e-6 relative to the fp32 dot
 * product; a bf16 K_imp is exact in TF32 and needs no split); rows with
 * massive ties are redone with fp32 FMA scores.  Always
 * one selection per query head. */
TB_API tb_status tb_select_prefill(tb_ctx* ctx, int layer, const void* q_imp_rows, int row0, int nrows,
                                   uint32_t* row_masks, int words_per_row, void* stream);

/* a8 — TokenSelect soft voting: votes[b][t] = sum_h softmax_t(q[b][h] . K[b][g(h)][t] / sqrt(D))
 * over t < len[b] (fp32), written to `votes` ([B][max_len]).  Select with
 * tb_select(rows_per_seq = 1) and attend with TB_MASK_SHARED. */
TB_API tb_status tb_softvote_scores(tb_ctx* ctx, int layer, const void* q, float* votes, void* stream);

/* ---- amortised selection ----------------------------------------------------
 * TokenButler abstract (importance predicted at intervals, neighbouring tokens
 * fetched) and TokenSelect README ("Selection Cache": consecutive similar
 * queries share selection results).  The pages fix none of the parameters.
 * With a cache bound to a layer and tb_set_reuse(interval > 0), every decode
 * step of that layer decides per selection row (query head, or KV group with
 * TB_BUTLER_GROUP) whether to reuse the row's cached selection:
 *   reuse  iff  the row takes a real top-k now (0 < k < candidates), the
 *               cache holds a top-k selected at length len0 > 0,
 *               len - len0 <= interval, and
 *               cos(q_hat_now, q_hat_cached) >= tau (fp32; for a group, its
 *               heads' importance queries summed in head order).
 * A reused row's set is the cached top-k (the cached mask inside
 * [sink, len0 - window)), widened by `radius` tokens on each side, kept inside
 * [sink, len - window), plus the current sink and window; its scores and
 * selection are not computed (a KV group whose rows all reuse is not scored).
 * Other rows select afresh and refill the cache.  The count check of reused
 * rows is skipped (their size is the cached top-k's). */

/* Bytes of one layer's selection cache for `cfg`. */
TB_API tb_status tb_selection_cache_size(const tb_config* cfg, size_t* bytes);
/* Bind a caller-owned, zero-filled, 256-byte aligned device buffer of at least
 * tb_selection_cache_size bytes as layer `layer`'s selection cache (NULL
 * unbinds).  TB_ERR_UNSUPPORTED for TB_SOFTVOTE. */
TB_API tb_status tb_bind_selection_cache(tb_ctx* ctx, int layer, void* cache, size_t bytes);
/* Reuse parameters: tau in [-1, 1], interval >= 0 tokens (0 turns reuse off),
 * radius in [0, 31]. */
TB_API tb_status tb_set_reuse(tb_ctx* ctx, float tau, int interval, int radius);

/* Copy the selection masks of the last sparse tb_decode_step, [B][rows][max_len/32]
 * uint32 (rows: Hq, Hkv with TB_BUTLER_GROUP, 1 with TB_SOFTVOTE), into a caller device buffer
 * of >= `bytes` bytes (stream-ordered; words past ceil(len/32) are stale). */
TB_API tb_status tb_copy_step_masks(tb_ctx* ctx, uint32_t* dst, size_t bytes, void* stream);

/* Failure-detection self-test (no counterpart on the pages).  Launches one
 * CTA that waits on an mbarrier expecting one arrival, with the same bounded
 * wait the pipelined kernels use (the tensor-core K_imp projection).  With
 * `arrive` != 0 the CTA arrives itself and the wait completes; with 0 nothing
 * arrives, the wait gives up after `cycles` SM cycles (1 .. 2e10) and sets
 * TB_DEV_ERR_TIMEOUT in the status word read by tb_check_status.  Neither
 * case faults, traps or hangs; the context stays usable.  TB_ERR_INVALID_ARG
 * for a NULL context or `cycles` out of range. */
TB_API tb_status tb_selftest_bounded_wait(tb_ctx* ctx, long long cycles, int arrive, void* stream);

/* ---- allocation-free attention ---------------------------------------------
 * The model card and the papers have no counterpart to this entry point; it
 * exists for callers that cannot allocate device memory (a serving loop with
 * a fixed memory budget that forbids allocation after start-up, a plug-in
 * whose host process owns all device memory, a runtime that only hands out
 * streams).  It computes exactly what tb_sparse_attn computes, without a
 * tb_ctx or a workspace: its split-K partials live in a static device array
 * of TB_STATIC_SCRATCH_BYTES inside the library, held by every GPU that
 * loads the library until the process exits.
 *   - `cache` describes the caller's K/V caches and lengths (host array);
 *     q, mask, mask_mode, out and lse are as for tb_sparse_attn.
 *   - TB_ERR_CAPACITY when the partials of the request (B * Hq * splits *
 *     (D + 2) floats) would not fit in the static array; TB_ERR_SHAPE when
 *     B * Hkv * max_len >= 2^31 or B * Hq * max_len >= 2^40 (the limits of a
 *     context); nothing is launched in either case.  The split count is the
 *     one tb_sparse_attn picks for the same lengths.
 *   - The first call on a device looks up the array's device address (with
 *     that device current); make that first call before any stream capture.
 *     The address is kept until the process exits: after cudaDeviceReset of
 *     a device, do not call this entry point on that device again.
 *   - All calls share the array and it keeps the last call's contents; calls
 *     that overlap on the GPU (several streams or threads) race on it.
 *   - It allocates nothing and calls no allocating routine. */
#define TB_STATIC_SCRATCH_BYTES (8u << 20)

typedef struct tb_cache_view {
  const void* k_cache;        /* [B][Hkv][max_len][D] device, kv_dtype          */
  const void* v_cache;        /* [B][Hkv][max_len][D] device, kv_dtype          */
  int batch, n_q_heads, n_kv_heads, head_dim, max_len, kv_dtype;
  const int32_t* lens_host;   /* [B] host: tokens per sequence                  */
} tb_cache_view;

TB_API tb_status tb_sparse_attn_static(const tb_cache_view* cache, const void* q, const uint32_t* mask,
                                       int mask_mode, void* out, float* lse, void* stream);

/* ---- Sequence-sharded decode (one long sequence over several ranks).
 * Beyond the pages, which decode on one device: each rank's context holds,
 * for every sequence, the contiguous global tokens [t0, t0 + len[b]) of its
 * caches (ranks in token order; appends go to the rank holding the end).
 * One step selects exactly the one-device set (model card "Method": top-x
 * under the global budget k = min(floor(P * L / 100), candidates), sink,
 * window, ties to the lower index) and merges the ranks' attention over
 * their parts by log-sum-exp.  Per layer and step, on every rank:
 *   tb_shard_set(layer, t0, global lengths)
 *   tb_score(...)                          local scores (rows: Hq, or Hkv with TB_BUTLER_GROUP)
 *   for pass in 0, 1:  tb_shard_hist -> sum the histograms over ranks -> tb_shard_pick(n_ranks = 1)
 *   pass 2:            tb_shard_hist -> gather the histograms in rank order -> tb_shard_pick(R, rank)
 *   tb_shard_mask                          this rank's mask words
 *   tb_sparse_attn_partial                 fp32 partial output and lse
 *   gather the partials in rank order -> tb_merge_partials
 * The collectives are the caller's (NCCL through torch.distributed in the
 * Python binding).  TB_ERR_UNSUPPORTED for TB_SOFTVOTE.  Buffers (device,
 * caller-owned):
 *   hist   [B*rows][2048] uint32 (pass 2: gathered [R][B*rows][2048])
 *   state  [B*rows][4] uint32: threshold key, counts, mode, quota
 *   mask   [B][rows][max_len/32] uint32 (words of this rank's local tokens)
 *   part   [B*Hq*D + B*Hq] fp32: output rows, then natural-log lse
 * A summed histogram holding fewer keys than the budget sets
 * TB_DEV_ERR_COUNT and leaves that row without its top-k. */
TB_API tb_status tb_shard_set(tb_ctx* ctx, int layer, int t0, const int32_t* global_lens_host);
/* zeroes `hist` and accumulates this rank's histogram of radix digit `pass`
 * (0: top 11 bits of the order key, 1: next 11, 2: low 10) over its
 * candidates, restricted by `state` to the digits found so far (pass > 0) */
TB_API tb_status tb_shard_hist(tb_ctx* ctx, int layer, const float* scores, int pass, const uint32_t* state,
                               uint32_t* hist, void* stream);
/* from the histogram summed over ranks (passes 0, 1; n_ranks = 1) or the
 * gathered per-rank histograms (pass 2; n_ranks = R, this rank's index),
 * the row's digit of the k-th largest key; pass 2 also sets the quota of
 * keys equal to the threshold this rank keeps */
TB_API tb_status tb_shard_pick(tb_ctx* ctx, int layer, int pass, const uint32_t* hist, int n_ranks, int rank,
                               uint32_t* state, void* stream);
TB_API tb_status tb_shard_mask(tb_ctx* ctx, int layer, const float* scores, const uint32_t* state, uint32_t* mask,
                               void* stream);
/* tb_sparse_attn writing fp32 output rows and lse into `part` (layout above) */
TB_API tb_status tb_sparse_attn_partial(tb_ctx* ctx, int layer, const void* q, const uint32_t* mask, int mask_mode,
                                        float* part, void* stream);
/* out[b][h] = sum_r exp(lse_r - lse) o_r over `n_parts` consecutive `part`
 * blocks (lse_r = -inf: no weight; all empty: zero output, lse -inf);
 * `lse` [B][Hq] may be NULL */
TB_API tb_status tb_merge_partials(tb_ctx* ctx, const float* parts, int n_parts, void* out, float* lse,
                                   void* stream);

/* Tracing: when `events` is non-NULL, tb_decode_step records the six
 * cudaEvent_t events[0..5] on its stream before the append, after the
 * append, after scoring, after selection, after the split attention kernel
 * and after the combine (points that a layer skips are recorded at the same
 * place).  `n_events` must be 6; NULL disables tracing. */
TB_API tb_status tb_trace_events(tb_ctx* ctx, void* const* events, int n_events);

/* Number of kernel launches this context has issued (a running total). */
TB_API tb_status tb_launch_count(const tb_ctx* ctx, uint64_t* count);

/* After a synchronisation: reads and clears the device status word.
 * Returns TB_ERR_DEVICE_STATUS if any bit was set (*flags gets them). */
TB_API tb_status tb_check_status(tb_ctx* ctx, uint32_t* flags);

TB_API const char* tb_status_string(tb_status s);
TB_API void tb_destroy(tb_ctx* ctx);

#ifdef __cplusplus
}
#endif

#endif /* TB_H */
