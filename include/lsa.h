/*
 * lsa.h -- C ABI of liblsa.so: one DeepSeek-Sparse-Attention (DSA) decode step
 * on NVIDIA B200 (sm_100a), and its causal prefill variant.
 *
 * What the step computes (sources are the pages this library restates):
 *
 *   1. Lightning-indexer scan.  Before each DSA layer a lightning indexer scores
 *      every cached token of the sequence and the layer attends only the k best
 *      (k = 2048 in production) -- MLI "Multi-layer Indexer" abstract
 *      (zhuanzhiai.com), sentence 2.  At long context this scan is where decode
 *      time goes (same abstract, sentence 3).  The score of cached token s for a
 *      query row is DSA's lightning-indexer form
 *          I(s) = sum_{h < H_I} w[h] * ReLU( sum_{d < d_I} q_idx[h][d] * K[s][d] )
 *      (DeepSeek-V3.2-Exp technical report, listed as a source on the LeanSparse
 *      episode page).  FP8 indexer keys carry a per-token scale:
 *      K[s][d] = scale[s] * e4m3(K[s][d]) (the compact indexer keys of the
 *      LeanSparse episode page).
 *   2. Top-k: the k highest scores of each row; equal scores go to the lower
 *      position; -inf and NaN are never selected.
 *   3. Sparse MQA over the selected rows only (what is read shrinks, what is
 *      stored does not: LeanSparse episode page): for every head h,
 *          o[h] = sum_j softmax_j(scale * q[h] . KV[idx_j]) * KV[idx_j][0:D_v]
 *      and lse[h] = log sum_j exp(scale * q[h] . KV[idx_j]).
 *   Prefill: a chunk of query rows at positions p_i scores the cache under a
 *   causal mask (s visible iff s <= p_i), then steps 2-3 run per row (the
 *   prefill workspace concern of the LeanSparse episode page).
 *
 * Conventions (all entry points):
 *   - Every pointer argument named as "device" is a CUDA device pointer on the
 *     current device; structs (lsa_dims, lsa_cache) live in host memory and are
 *     read during the call only.  The caller owns every buffer.
 *   - The library never allocates device memory and never synchronises the
 *     stream, except lsa_read_device_status and lsa_get_device_status, which
 *     do both a copy and a stream synchronisation by design.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream).  A call returns after enqueueing.
 *   - Host-checkable argument errors return an error code and enqueue nothing.
 *   - Errors only the GPU can see (a block-table entry outside the pool, a
 *     sequence length above max_len) make the kernels skip the bad access, write
 *     NaN for affected outputs, and record the first such error in the
 *     workspace status word; read it with lsa_read_device_status.  Kernels never
 *     trap.
 *   - Cache addressing: positions are logical token positions.  Paged caches
 *     (block_size > 0) map position p of sequence b to the stored row
 *     block_table[b][p / block_size] * block_size + p % block_size.  Contiguous
 *     caches (block_size == 0) map it to row b * max_len + p.
 *   - Workspace: `ws` is a device buffer of at least lsa_workspace_size(...)
 *     bytes, 256-byte aligned.  Its first 256 bytes hold the status word; zero
 *     them once after allocating (e.g. allocate zero-filled).  Calls that share
 *     one workspace must be ordered on one stream.
 */
#ifndef LSA_H_
#define LSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define LSA_VERSION 1

typedef struct CUstream_st* lsa_stream_t; /* same handle type as cudaStream_t */

typedef enum {
  LSA_OK = 0,
  LSA_ERR_INVALID_ARG = 1, /* host-checkable argument error; nothing enqueued */
  LSA_ERR_UNSUPPORTED = 2, /* valid but unsupported shape/dtype combination */
  LSA_ERR_WORKSPACE = 3,   /* ws NULL, misaligned or smaller than required */
  LSA_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch, attribute) */
  LSA_ERR_TIMEOUT = 5,     /* device: a bounded wait gave up (status word) */
  LSA_ERR_BOUNDS = 6       /* device: block id / length out of range (status word) */
} lsa_status;

typedef enum { LSA_F32 = 0, LSA_BF16 = 1, LSA_FP8_E4M3 = 2 } lsa_dtype;

/* Shapes and element types of the step; validated on every call. */
typedef struct {
  int32_t n_idx_heads;   /* H_I: indexer heads (1..64)                              */
  int32_t idx_dim;       /* d_I: indexer head dim (multiple of 8, 8..256)           */
  int32_t n_heads;       /* H: attention query heads sharing one KV row (MQA)       */
  int32_t qk_dim;        /* D: KV row width = q width (multiple of 8, <= 1024)      */
  int32_t v_dim;         /* D_v <= D: the value is the first D_v columns of the row */
  int32_t top_k;         /* k: tokens kept per query row (1..8192)                  */
  int32_t block_size;    /* tokens per cache block, 0 = contiguous caches           */
  float softmax_scale;   /* logit scale of the sparse attention                     */
  int32_t act_dtype;     /* q_idx, q, kv and out: LSA_F32 or LSA_BF16               */
  int32_t idx_key_dtype; /* indexer keys: LSA_F32, LSA_BF16 or LSA_FP8_E4M3         */
} lsa_dims;

/* Caller-owned caches of one layer (device pointers). */
typedef struct {
  const void* idx_keys;        /* [n_blocks, bs, d_I] or [batch, max_len, d_I], idx_key_dtype */
  const float* idx_key_scales; /* FP8 keys only: [n_blocks, bs] or [batch, max_len]; else NULL */
  const void* kv;              /* [n_blocks, bs, D] or [batch, max_len, D], act_dtype; may be
                                  NULL for calls that do not read it                             */
  const int32_t* block_table;  /* [batch, max_blocks_per_seq] (paged) or NULL (contiguous)      */
  int32_t max_blocks_per_seq;  /* row stride of block_table (paged)                             */
  int64_t n_blocks;            /* physical blocks in each pool (paged); bounds for block ids    */
  int64_t max_len;             /* upper bound of seq_lens; contiguous: row stride in tokens     */
  const int32_t* seq_lens;     /* [batch] valid cached tokens per sequence (device)             */
  int32_t batch;               /* sequences                                                     */
} lsa_cache;

/* Operation selector for lsa_workspace_size. */
typedef enum {
  LSA_OP_SCORES = 0,
  LSA_OP_TOPK = 1,
  LSA_OP_ATTN = 2,
  LSA_OP_DECODE_STEP = 3,
  LSA_OP_DECODE_STEP_FUSED = 4, /* lsa_launch_count only: lsa_decode_step with LSA_STEP_FUSED */
  LSA_OP_DECODE_LAYERS = 5      /* lsa_decode_layers (lsa_workspace_size; see lsa_launch_count) */
} lsa_op;

/* Flags of lsa_decode_step. */
#define LSA_STEP_UNFUSED 0 /* scan, top-k, attention as separate launches     */
#define LSA_STEP_FUSED 1   /* the whole step in one cooperative launch        */

/*
 * Bytes of workspace `op` needs for `rows` query rows whose score rows hold
 * `max_len` entries (0 on invalid arguments).  For LSA_OP_TOPK only d->top_k
 * is read (the k of the lsa_topk call).
 */
size_t lsa_workspace_size(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t op);

/*
 * Lightning-indexer scores for `rows` query rows (step 1).
 *   row_seq  [rows] device: sequence of each row, or NULL (row r -> sequence r).
 *   row_pos  [rows] device: causal position of each row (prefill), or NULL
 *            (decode: all seq_lens[b] positions are visible).
 *   q_idx    [rows, H_I, d_I] device, act_dtype (bf16 or f32).
 *   w        [rows, H_I] device fp32.
 *   scores   [rows, ld] device fp32 out: I(s) for visible s; -inf for masked
 *            positions (s > p_i) and for s in [seq_len, ld).  ld >= max_len.
 * Errors: LSA_ERR_INVALID_ARG (NULL pointers, bad dims, ld < max_len),
 *         LSA_ERR_UNSUPPORTED, LSA_ERR_WORKSPACE, LSA_ERR_CUDA.
 */
lsa_status lsa_indexer_scores(const lsa_dims* d, const lsa_cache* c, int32_t rows,
                              const int32_t* row_seq, const int32_t* row_pos,
                              const void* q_idx, const float* w, float* scores, int64_t ld,
                              void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * Top-k of each score row (step 2), exact on the fp32 values.
 *   scores    [rows, ld] device fp32.
 *   valid_len [rows] device: entries [0, valid_len[r]) take part, or NULL
 *             (every row has n_cols entries).  valid_len[r] is clamped to n_cols.
 *   idx       [rows, k] device int32 out: positions of the min(k, #selectable)
 *             largest entries (ties -> lower position; -0.0 == +0.0; -inf and
 *             NaN never selected), sorted ascending, padded with -1.
 * Errors: LSA_ERR_INVALID_ARG, LSA_ERR_WORKSPACE, LSA_ERR_CUDA.
 */
lsa_status lsa_topk(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len,
                    int64_t n_cols, int32_t k, int32_t* idx,
                    void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * Sparse MQA over selected rows (step 3).
 *   row_seq [rows] device or NULL (row r -> sequence r).
 *   q       [rows, H, D] device, act_dtype.
 *   idx     [rows, d->top_k] device int32: positions (-1 = none; any order).
 *   out     [rows, H, D_v] device, act_dtype out; rows with no position give 0.
 *   lse     [rows, H] device fp32 out (natural log; -inf for empty rows), or NULL.
 * Positions >= the sequence's length are a device error (LSA_ERR_BOUNDS).
 */
lsa_status lsa_sparse_attn_decode(const lsa_dims* d, const lsa_cache* c, int32_t rows,
                                  const int32_t* row_seq, const void* q, const int32_t* idx,
                                  void* out, float* lse,
                                  void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * One decode step for every sequence of the cache (rows = c->batch, row b ->
 * sequence b): scores -> top-k -> sparse attention.
 *   q_idx [B, H_I, d_I], w [B, H_I] fp32, q [B, H, D]: device inputs.
 *   out [B, H, D_v], lse [B, H] (or NULL): device outputs.
 *   idx_out [B, k] device int32 or NULL: the selection, if wanted.
 *   flags: LSA_STEP_UNFUSED: the scan, the top-k and the attention are
 *            separate launches (3-5 kernels, see lsa_launch_count).
 *          LSA_STEP_FUSED: the same three stages in ONE cooperative launch of
 *            one CTA per SM, with grid-wide barriers (bounded waits) between
 *            them (the optional fused decode kernel of the MLI page, a
 *            single persistent launch here).  It runs the same CTA code as the
 *            separate launches, so its results are bitwise those of
 *            LSA_STEP_UNFUSED.  It applies when the tensor-core scan, the
 *            three-pass top-k (c->max_len <= 2^19) and the tensor-core
 *            attention all apply and every CTA of the grid fits on the device
 *            at once; otherwise the step silently takes the separate launches.
 *            A barrier that times out records LSA_ERR_TIMEOUT in the status word.
 * Workspace: lsa_workspace_size(d, B, c->max_len, LSA_OP_DECODE_STEP) (either flag).
 */
lsa_status lsa_decode_step(const lsa_dims* d, const lsa_cache* c, const void* q_idx,
                           const float* w, const void* q, void* out, float* lse,
                           int32_t* idx_out, int32_t flags,
                           void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * lsa_decode_step that also records CUDA events on `stream` at its phase
 * boundaries, for profiling: events[0] before the scan, events[1] after the
 * scan, events[2] after the top-k, events[3] after the sparse attention.
 * `events` is an array of 4 cudaEvent_t (NULL entries are skipped) or NULL.
 * Results, workspace and errors as lsa_decode_step (LSA_ERR_CUDA if an event
 * record fails).
 */
lsa_status lsa_decode_step_profiled(const lsa_dims* d, const lsa_cache* c, const void* q_idx,
                                    const float* w, const void* q, void* out, float* lse,
                                    int32_t* idx_out, int32_t flags, void* ws, size_t ws_bytes,
                                    lsa_stream_t stream, void* const* events);

/* Routes of lsa_decode_layers: which indexer layer's selection a layer attends. */
#define LSA_ROUTE_OWN 0  /* the latest indexer layer at or before it (IndexCache; DSA at retention 1) */
#define LSA_ROUTE_PREV 1 /* the latest indexer layer before it (Multi-layer Indexer); layer 0: its own */

/*
 * Several DSA layers of one decode step ("Multi-layer Indexer" abstract,
 * zhuanzhiai.com, sentences 4-5 and 8-9: IndexCache keeps an indexer on a
 * fraction 1/r of the layers and the others reuse the latest selection; MLI
 * lets a layer attend the previous indexer layer's selection, so its own
 * indexer runs alongside its attention).
 *   n_layers >= 1 layers; every array argument is a HOST array of n_layers
 *   entries holding device pointers:
 *     caches[l]  layer l's cache: the same batch B, max_len, seq_lens, block
 *                table and block size for every layer, its own idx_keys,
 *                idx_key_scales (FP8) and kv.
 *     q_idx[l] [B, H_I, d_I], w[l] [B, H_I] fp32: read only for the layers
 *                that keep an indexer.
 *     q[l] [B, H, D]: layer l's attention query.
 *     out[l] [B, H, D_v], lse[l] [B, H] fp32 (lse may be NULL, or lse[l] NULL).
 *   retention r >= 1: layers 0, r, 2r, ... keep an indexer.
 *   route: LSA_ROUTE_OWN or LSA_ROUTE_PREV (above).
 *   idx_out: NULL or device int32 [n_layers, B, k]: the selection each layer
 *            attended (sorted ascending, -1 padded, as lsa_topk).
 * Order on `stream`: layer l+1 starts after layer l's attention has finished
 * (a layer's queries depend on the previous layer's output).  Within a layer
 * that keeps an indexer, LSA_ROUTE_OWN runs scan -> top-k -> attention as
 * lsa_decode_step does; LSA_ROUTE_PREV launches the attention (on the earlier
 * selection) first and the layer's scan as its programmatic dependent, so
 * the scan runs on the SMs the attention leaves free while it runs (MLI
 * abstract: each indexer runs concurrently with its layer's attention), then
 * the top-k into a second selection buffer.
 * Results per layer equal lsa_decode_step / lsa_sparse_attn_decode on the
 * routed selection.
 * Workspace: lsa_workspace_size(d, B, max_len, LSA_OP_DECODE_LAYERS).
 * Errors: LSA_ERR_INVALID_ARG for n_layers < 1, retention < 1, an unknown
 * route, layers whose batch, max_len, seq_lens or block table differ from
 * layer 0's, or a missing or misaligned pointer; nothing is launched then.
 */
lsa_status lsa_decode_layers(const lsa_dims* d, int32_t n_layers, const lsa_cache* caches,
                             const void* const* q_idx, const float* const* w, const void* const* q,
                             void* const* out, float* const* lse, int32_t retention, int32_t route,
                             int32_t* idx_out, void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * Exact indexer scores of given candidate positions (the second stage of the
 * two-stage search below): for row r and entry j < n_cand,
 *   scores[r][j] = I(cand[r][j]) over the cache's own (original) keys,
 * the score of step 1 at that position.
 *   row_seq, row_pos, q_idx, w: as lsa_indexer_scores.
 *   cand   [rows, n_cand] device int32: positions (any order, -1 = none).
 *   scores [rows, ld] device fp32 out, ld >= n_cand: -inf for -1 entries and
 *          for [n_cand, ld); NaN (and LSA_ERR_BOUNDS in the status word) for a
 *          position outside the row's visible range or a bad block.
 * Supported: bf16 keys and queries, 64 x 128 indexer heads (else
 * LSA_ERR_UNSUPPORTED); any block size.  Workspace: 256 bytes (status word).
 */
lsa_status lsa_candidate_scores(const lsa_dims* d, const lsa_cache* c, int32_t rows,
                                const int32_t* row_seq, const int32_t* row_pos,
                                const void* q_idx, const float* w, const int32_t* cand,
                                int32_t n_cand, float* scores, int64_t ld,
                                void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * Two-stage selection (LeanSparse episode page, summary: during decode, search
 * compact indexer keys and fetch only a short list of the originals to rank
 * exactly).  For each query row:
 *   1. compact scores: step 1 over the compact keys, e4m3 with one fp32 scale
 *      per token (K ~ scale * e4m3, the FP8 key form);
 *   2. the short list: the n_cand positions with the highest compact scores
 *      (ties to the lower position);
 *   3. their exact scores over the original bf16 keys of `c`;
 *   4. the k = d->top_k best of the list by exact score (ties to the lower
 *      position), sorted ascending, -1 padded -> idx [rows, k].
 * The original keys are read only at the n_cand listed positions: per row the
 * bytes of the scan drop from L * 256 to L * 132 + n_cand * 256.
 *   c               the cache with its original bf16 keys (d->idx_key_dtype =
 *                   LSA_BF16); kv is not read.
 *   compact_keys    e4m3 bytes in the layout of c->idx_keys (1 byte per dim).
 *   compact_scales  fp32, one per token, in the layout of FP8 key scales.
 *   n_cand          >= k; with n_cand >= the row's length the result is the
 *                   exact top-k of step 2.
 * Workspace: lsa_two_stage_workspace_size(d, rows, c->max_len, n_cand).
 * Errors: LSA_ERR_INVALID_ARG (n_cand < k, missing or misaligned pointers),
 * LSA_ERR_UNSUPPORTED (other than bf16 keys and queries with 64 x 128 indexer
 * heads and block sizes that are multiples of 64), LSA_ERR_WORKSPACE,
 * LSA_ERR_CUDA.  Launches: scan, top-k (2), candidate scores, top-k (2), and
 * one kernel that maps list entries to positions.
 */
size_t lsa_two_stage_workspace_size(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t n_cand);
lsa_status lsa_two_stage_select(const lsa_dims* d, const lsa_cache* c, const void* compact_keys,
                                const float* compact_scales, int32_t rows, const int32_t* row_seq,
                                const int32_t* row_pos, const void* q_idx, const float* w,
                                int32_t n_cand, int32_t* idx, void* ws, size_t ws_bytes,
                                lsa_stream_t stream);

/*
 * Block-level selection (SparDA abstract, page 4 of the sources: the selector
 * picks the KV blocks a layer needs, and a forecast of the next layer's blocks
 * lets their host-to-device copy overlap the current layer's work).
 *
 * lsa_block_select: for each row, the score of every block of block_size
 * consecutive positions is the largest score among its positions below
 * valid_len[r] (or n_cols; NaN ignored, -inf for a block with none); the
 * n_sel best blocks (ties to the lower block; blocks scoring -inf never) go
 * to kept [rows, n_sel] device int32, ascending, -1 padded.
 *   scores [rows, ld] device fp32 (e.g. lsa_indexer_scores' output).
 * Workspace: lsa_block_select_workspace_size(rows, n_cols, block_size, n_sel).
 * Launches: the block maximum, then the top-k's (2).
 */
size_t lsa_block_select_workspace_size(int32_t rows, int64_t n_cols, int32_t block_size, int32_t n_sel);
lsa_status lsa_block_select(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len,
                            int64_t n_cols, int32_t block_size, int32_t n_sel, int32_t* kept,
                            void* ws, size_t ws_bytes, lsa_stream_t stream);

/*
 * lsa_stage_blocks: copies every row's kept blocks from the cache's KV into a
 * staging pool, one launch of one CTA per (row, kept block):
 *   c->kv may be device memory or page-locked host memory the device can map
 *     (an offloaded cache: the copy then reads it across the host link; issue
 *     the call on a copy-side stream to overlap it with other work).  Other
 *     host memory returns LSA_ERR_INVALID_ARG.
 *   row_seq, row_pos: as lsa_indexer_scores (a causal row keeps the positions
 *     up to its own).
 *   kept [rows, n_sel] device: block ids as lsa_block_select gives them.
 *   block_size: positions per block; for a paged cache it must equal
 *     d->block_size (a kept block is one page).
 *   staged_kv [rows * n_sel, block_size, D] device, act_dtype out: staged block
 *     r * n_sel + i holds kept block i of row r (rows past the sequence zero).
 *   staged_table [rows, n_sel] device int32 out: r * n_sel + i, or -1 where
 *     nothing was kept.
 *   staged_idx [rows, n_sel * block_size] device int32 out: the positions of the
 *     staged sequence the row attends: i * block_size + t for every kept
 *     position, -1 elsewhere.
 * The row then attends its kept blocks with lsa_sparse_attn_decode on a cache
 * over the staging pool (kv = staged_kv, block_table = staged_table,
 * block_size = block_size, max_blocks_per_seq = n_sel, n_blocks = rows *
 * n_sel, max_len = n_sel * block_size, seq_lens = that length per row, batch
 * = rows), d->top_k = n_sel * block_size, and idx = staged_idx.
 * Workspace: 256 bytes (the status word; a block id outside the pool records
 * LSA_ERR_BOUNDS).
 */
lsa_status lsa_stage_blocks(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                            const int32_t* row_pos, const int32_t* kept, int32_t n_sel, int32_t block_size, void* staged_kv,
                            int32_t* staged_table, int32_t* staged_idx, void* ws, size_t ws_bytes,
                            lsa_stream_t stream);

/*
 * Prefill of a chunk of query rows through several layers with each layer's
 * history streamed through two alternating device buffers (LeanSparse episode
 * page, summary: during prefill, stream each layer's history through two GPU
 * buffers that alternate, so the prefill does not need every layer's KV
 * resident, nor the large temporary workspace that forces).  Layer l runs on
 * buffer l % 2 while the copy of layer l+1's history into the other buffer
 * proceeds on the copy stream.
 *   caches[l]  (HOST array of n_layers) layer l's cache of ONE sequence
 *              (batch 1, contiguous: d->block_size = 0), every layer with the
 *              same max_len = L (the visible sequence, history and chunk) and
 *              seq_lens; idx_keys on the device (the indexer keys stay on the
 *              GPU); kv = the layer's history rows [0, hist_len), in
 *              page-locked host memory (an offloaded cache) or device memory.
 *   chunk_kv[l] device [L - hist_len, D]: the chunk's own KV rows of layer l.
 *   rows, row_pos [rows] device: the chunk's query rows and their positions.
 *   q_idx[l], w[l], q[l], out[l], lse[l] (lse may be NULL or hold NULL),
 *   idx_out[l] ([rows, k], may be NULL or hold NULL): per layer, as
 *              lsa_indexer_scores / lsa_topk / lsa_sparse_attn_decode.
 *   row_block  rows scored, selected and attended at a time: the score
 *              workspace is row_block x L fp32 instead of rows x L.
 *   kv_buf[2]  device [L, D] each: the alternating history buffers.
 *   compute, copy: two streams (the copies run on `copy`, everything else on
 *              `compute`); events[4]: cudaEvent_t created by the caller
 *              (timing disabled is best): buffer 0 and 1 filled, buffer 0 and 1
 *              released.  The call enqueues and returns; `compute` holds the
 *              last layer's work.
 * Each layer's results equal lsa_indexer_scores -> lsa_topk -> lsa_sparse_attn_decode
 * on its whole cache (bit for bit with row_block >= rows).
 * Workspace: lsa_prefill_layers_workspace_size(d, rows, L, row_block).
 */
size_t lsa_prefill_layers_workspace_size(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t row_block);
lsa_status lsa_prefill_layers(const lsa_dims* d, int32_t n_layers, const lsa_cache* caches, int64_t hist_len,
                              const void* const* chunk_kv, int32_t rows, const int32_t* row_pos,
                              const void* const* q_idx, const float* const* w, const void* const* q,
                              void* const* out, float* const* lse, int32_t* const* idx_out, int32_t row_block,
                              void* const* kv_buf, void* ws, size_t ws_bytes, lsa_stream_t compute,
                              lsa_stream_t copy, void* const* events);

/*
 * Copies the workspace status word to *status (an lsa_status value), clears it,
 * and synchronises `stream`.  Returns LSA_ERR_CUDA if a CUDA call fails.
 */
lsa_status lsa_read_device_status(void* ws, int32_t* status, lsa_stream_t stream);

/*
 * The same read as a single status: the workspace status word (an lsa_status
 * value, LSA_OK if no kernel recorded an error), which is cleared; or
 * LSA_ERR_INVALID_ARG for a NULL workspace, or LSA_ERR_CUDA if a CUDA call of
 * the read fails.  Synchronises `stream` like lsa_read_device_status.
 */
lsa_status lsa_get_device_status(void* ws, lsa_stream_t stream);

/*
 * Top-k without a workspace argument, for callers that cannot allocate device
 * memory where they call it: a plugin host whose enqueue path forbids
 * allocation, a runtime whose device memory is all pre-reserved by another
 * allocator, or a latency-critical loop that cannot pay for cudaMalloc's
 * implicit synchronisation.  (The pages describe no such entry point; it is
 * an addition of this library.)
 *   Same arguments, results and errors as lsa_topk, minus ws / ws_bytes.
 *   Scratch: a 4 MiB static device array inside liblsa.so, held by every GPU
 *   that loads the library until the process exits.  Sizes whose top-k scratch
 *   (lsa_workspace_size with d->top_k = k, LSA_OP_TOPK) exceeds 4 MiB less
 *   256 bytes return LSA_ERR_UNSUPPORTED (about 40 rows of 128K scores fit).
 *   Allocates nothing: no cudaMalloc / cudaFree; the histograms are cleared
 *   with cudaMemsetAsync on `stream` at every call.
 *   The first call on a device looks up the array's device address (once per
 *   device, with that device current); make that first call before any stream
 *   capture.
 *   Every call shares the one array: calls that overlap on the GPU (different
 *   streams, or different host threads on one device) race and give wrong
 *   results.  Device-side error reports of this entry point are not readable
 *   through lsa_read_device_status.
 */
lsa_status lsa_topk_noalloc(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len,
                            int64_t n_cols, int32_t k, int32_t* idx, lsa_stream_t stream);

/*
 * Number of kernel launches `op` enqueues for `rows` query rows with score rows
 * of `max_len` entries (`causal` != 0: prefill rows with positions), assuming
 * 16-byte aligned buffers.  A planning aid for launch accounting and graph
 * capture; runtime memsets are not counted.  LSA_OP_DECODE_STEP_FUSED gives
 * 1 when the fused step applies to these shapes, else the separate launches'
 * count (the device can still refuse the cooperative launch at run time, in
 * which case the step falls back to them).  LSA_OP_DECODE_LAYERS gives -1:
 * lsa_decode_layers enqueues, per layer, the launches of LSA_OP_DECODE_STEP
 * for a layer that keeps an indexer and of LSA_OP_ATTN for the others.  -1 on
 * invalid arguments.
 */
int32_t lsa_launch_count(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t op, int32_t causal);

/* Static description of a status code. */
const char* lsa_status_string(lsa_status s);

/* LSA_VERSION of the built library. */
int32_t lsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* LSA_H_ */
