// C ABI of liblsa.so (declared in include/lsa.h): argument validation,
// workspace layout and kernel dispatch.  No allocation, no synchronisation
// (except lsa_read_device_status).
#include <cuda_runtime.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "common.cuh"
#include "internal.h"
#include "lsa.h"
#ifdef LSA_TEST_HOOKS
#include "lsa_test.h"
#endif

namespace lsa {
namespace {

constexpr size_t kAlign = 256;

inline size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Rows at least this long take the split select in a decode step.
constexpr int64_t kSplitSelectMinCols = int64_t(1) << 18;

// Timing model of the MLI layer's scan split (measured on B200 at 1965 MHz): a
// tensor-core attention CTA takes about kAttnFixedUs plus kAttnChunkUs per
// 64-entry chunk, and a scan CTA streams one 128-token bf16 tile per
// kScanTileUs.  It only decides how many tiles the first scan launch takes.
constexpr double kAttnFixedUs = 21.0;
constexpr double kAttnChunkUs = 2.2;
constexpr double kScanTileUs = 0.72;
// The decode scan's pooled schedule (each CTA's even share of the first
// pool_static_pm thousandths of the tiles, then chunks of pool_chunk tiles
// from a counter) is exact but measured no faster than the static split at
// B = 32 (step 0.2231 against 0.2217 ms with 90 % static and chunks of 4;
// 0.2214 with 95 %) and slower for the FP8 keys at B = 4 (0.1524 against
// 0.1293 ms: every segment restages and converts the query and flushes the
// histogram).  The static split is the default; the test build can switch
// the pool on (lsa_test_set_scan_pool).  A value above 1000 means no pool.
constexpr int kPoolChunk = 4;
constexpr int kPoolStaticPm = 1001;

#ifdef LSA_TEST_HOOKS
// Test build only (liblsa_test.so, include/lsa_test.h): switches that tests
// set through lsa_test_set_hooks.  The product library has none of them, so
// nothing in a serving process (no environment variable, no call) can change
// its path or break its handoffs.
struct TestHooks {
  bool force_simt = false;                         // every call on the CUDA-core kernels
  int64_t split_select_min_cols = kSplitSelectMinCols;
  uint32_t scan_wait_extra = 0;                    // raises the decode step's scan-CTA count
  bool no_cluster_topk = false;                    // the collect + select top-k for every row length
  int pool_static_pm = kPoolStaticPm;              // > 1000: the decode scan without its pool
  int pool_chunk = kPoolChunk;
};
TestHooks g_hooks;
bool force_simt() { return g_hooks.force_simt; }
int64_t split_select_min_cols() { return g_hooks.split_select_min_cols; }
uint32_t test_scan_wait_extra() { return g_hooks.scan_wait_extra; }
bool allow_cluster_topk() { return !g_hooks.no_cluster_topk; }
int pool_static_pm() { return g_hooks.pool_static_pm; }
int pool_chunk() { return g_hooks.pool_chunk; }
#else
constexpr bool force_simt() { return false; }
constexpr int64_t split_select_min_cols() { return kSplitSelectMinCols; }
constexpr uint32_t test_scan_wait_extra() { return 0u; }
constexpr bool allow_cluster_topk() { return true; }
constexpr int pool_static_pm() { return kPoolStaticPm; }
constexpr int pool_chunk() { return kPoolChunk; }
#endif

bool valid_dims(const lsa_dims* d) {
  if (!d) return false;
  if (d->n_idx_heads < 1 || d->n_idx_heads > 64) return false;
  if (d->idx_dim < 8 || d->idx_dim > 256 || d->idx_dim % 8) return false;
  if (d->n_heads < 1 || d->n_heads > 4096) return false;
  if (d->qk_dim < 8 || d->qk_dim > 1024 || d->qk_dim % 8) return false;
  if (d->v_dim < 1 || d->v_dim > d->qk_dim) return false;
  if (d->top_k < 1 || d->top_k > (1 << 20)) return false;
  if (d->block_size < 0) return false;
  if (d->act_dtype != LSA_F32 && d->act_dtype != LSA_BF16) return false;
  if (d->idx_key_dtype != LSA_F32 && d->idx_key_dtype != LSA_BF16 && d->idx_key_dtype != LSA_FP8_E4M3)
    return false;
  if (!(d->softmax_scale == d->softmax_scale)) return false;
  return true;
}

bool valid_cache(const lsa_dims* d, const lsa_cache* c, bool need_keys, bool need_kv) {
  if (!c || !c->seq_lens || c->batch < 0 || c->max_len < 0) return false;
  if (d->block_size > 0) {
    if (!c->block_table || c->max_blocks_per_seq < 1 || c->n_blocks < 1) return false;
    if (static_cast<int64_t>(c->max_blocks_per_seq) * d->block_size < c->max_len) return false;
  }
  if (need_keys) {
    if (!c->idx_keys || !aligned16(c->idx_keys)) return false;
    if (d->idx_key_dtype == LSA_FP8_E4M3 && !c->idx_key_scales) return false;
  }
  if (need_kv && (!c->kv || !aligned16(c->kv))) return false;
  return true;
}

CacheView view(const lsa_dims* d, const lsa_cache* c) {
  CacheView v;
  v.idx_keys = c->idx_keys;
  v.idx_key_scales = c->idx_key_scales;
  v.kv = c->kv;
  v.block_table = c->block_table;
  v.max_blocks = c->max_blocks_per_seq;
  v.n_blocks = d->block_size > 0 ? c->n_blocks : 0;
  v.max_len = c->max_len;
  v.seq_lens = c->seq_lens;
  v.batch = c->batch;
  v.block_size = d->block_size;
  return v;
}

size_t scores_ws(int32_t rows, bool causal) { return align_up(scores_tc_ws_bytes(rows, causal)); }

size_t attn_ws(const lsa_dims* d, int32_t rows) {
  size_t a = attn_simt_ws_bytes(rows, d->n_heads, d->v_dim, d->top_k);
  size_t b = attn_tc_ws_bytes(rows, d->n_heads, d->qk_dim, d->v_dim, d->top_k);
  return align_up(a > b ? a : b);
}

inline int64_t score_ld(int64_t max_len) { return (max_len + 3) / 4 * 4; }

struct StepLayout {
  size_t scores_off, idx_off, inner_off, total;
};

StepLayout step_layout(const lsa_dims* d, int32_t rows, int64_t max_len) {
  StepLayout L;
  L.scores_off = kStatusBytes;
  L.idx_off = L.scores_off + align_up(static_cast<size_t>(rows) * score_ld(max_len) * 4);
  L.inner_off = L.idx_off + align_up(static_cast<size_t>(rows) * d->top_k * 4);
  size_t inner = topk_ws_bytes(rows, max_len, d->top_k);
  if (topk_v2_ok(max_len)) {  // the fused step keeps the top-k head and the attention partials together
    const size_t f = step_fused_ws_bytes(rows, max_len, d->top_k);
    if (f > inner) inner = f;
  }
  size_t a = attn_ws(d, rows);
  size_t s = scores_ws(rows, false);
  if (a > inner) inner = a;
  if (s > inner) inner = s;
  L.total = L.inner_off + align_up(inner);
  return L;
}

// Several layers (lsa_decode_layers): the scores, two selection buffers (the
// latest indexer selection and the one being made), the scan / top-k scratch
// and, apart from it, the attention's (the two run at once under the MLI route).
struct LayersLayout {
  size_t scores_off, sel_off[2], tk_off, tk_bytes, at_off, at_bytes, total;
};

LayersLayout layers_layout(const lsa_dims* d, int32_t rows, int64_t max_len) {
  LayersLayout L;
  const size_t sel = align_up(static_cast<size_t>(rows) * d->top_k * 4);
  L.scores_off = kStatusBytes;
  L.sel_off[0] = L.scores_off + align_up(static_cast<size_t>(rows) * score_ld(max_len) * 4);
  L.sel_off[1] = L.sel_off[0] + sel;
  L.tk_off = L.sel_off[1] + sel;
  size_t tk = topk_ws_bytes(rows, max_len, d->top_k);
  const size_t sc = scores_ws(rows, false);
  if (sc > tk) tk = sc;
  L.tk_bytes = align_up(tk);
  L.at_off = L.tk_off + L.tk_bytes;
  L.at_bytes = attn_ws(d, rows);
  L.total = L.at_off + L.at_bytes;
  return L;
}

// The two-stage search (lsa_two_stage_select): the compact scores, the
// candidate list, the candidates' exact scores, the chosen candidate entries,
// and the scratch of the scans and the two top-k calls.
struct TwoStageLayout {
  size_t cscores_off, cand_off, exact_off, slot_off, inner_off, inner_bytes, total;
  int64_t ld_c, ld_x;
};

TwoStageLayout two_stage_layout(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t n_cand) {
  TwoStageLayout L;
  const size_t R = static_cast<size_t>(rows);
  L.ld_c = score_ld(max_len);
  L.ld_x = score_ld(n_cand);
  L.cscores_off = kStatusBytes;
  L.cand_off = L.cscores_off + align_up(R * L.ld_c * 4);
  L.exact_off = L.cand_off + align_up(R * static_cast<size_t>(n_cand) * 4);
  L.slot_off = L.exact_off + align_up(R * L.ld_x * 4);
  L.inner_off = L.slot_off + align_up(R * static_cast<size_t>(d->top_k) * 4);
  size_t inner = topk_ws_bytes(rows, max_len, n_cand);
  const size_t t2 = topk_ws_bytes(rows, n_cand, d->top_k);
  const size_t sc = scores_ws(rows, true);
  if (t2 > inner) inner = t2;
  if (sc > inner) inner = sc;
  L.inner_bytes = align_up(inner);
  L.total = L.inner_off + L.inner_bytes;
  return L;
}

// Layer-streamed prefill (lsa_prefill_layers): the rows' sequence map (all
// zero), one block of rows' scores and selection, and the scan / top-k /
// attention scratch of a block.
struct PrefillLayout {
  size_t rowseq_off, scores_off, idx_off, inner_off, inner_bytes, total;
  int64_t ld;
};

PrefillLayout prefill_layout(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t row_block) {
  PrefillLayout L;
  const int32_t rb = row_block < rows ? row_block : rows;
  L.ld = score_ld(max_len);
  L.rowseq_off = kStatusBytes;
  L.scores_off = L.rowseq_off + align_up(static_cast<size_t>(rows) * 4);
  L.idx_off = L.scores_off + align_up(static_cast<size_t>(rb) * L.ld * 4);
  L.inner_off = L.idx_off + align_up(static_cast<size_t>(rb) * d->top_k * 4);
  size_t inner = topk_ws_bytes(rb, max_len, d->top_k);
  const size_t a = attn_ws(d, rb), sc = scores_ws(rb, true);
  if (a > inner) inner = a;
  if (sc > inner) inner = sc;
  L.inner_bytes = align_up(inner);
  L.total = L.inner_off + L.inner_bytes;
  return L;
}

lsa_status ws_check(void* ws, size_t have, size_t need) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) % kAlign) != 0) return LSA_ERR_WORKSPACE;
  if (have < need) return LSA_ERR_WORKSPACE;
  return LSA_OK;
}

inline lsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? LSA_OK : LSA_ERR_CUDA; }

inline DevStatus* status_of(void* ws) { return reinterpret_cast<DevStatus*>(ws); }

ScoresArgs scores_args(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                       const int32_t* row_pos, const void* q_idx, const float* w, float* scores, int64_t ld,
                       void* ws, void* inner_ws, size_t inner_bytes) {
  ScoresArgs a;
  a.cache = view(d, c);
  a.key_dtype = d->idx_key_dtype;
  a.q_dtype = d->act_dtype;
  a.H = d->n_idx_heads;
  a.dI = d->idx_dim;
  a.rows = rows;
  a.row_seq = row_seq;
  a.row_pos = row_pos;
  a.q_idx = q_idx;
  a.w = w;
  a.scores = scores;
  a.ld = ld;
  a.status = status_of(ws);
  a.plan_ws = inner_ws;
  a.plan_bytes = inner_bytes;
  a.hist12 = nullptr;
  return a;
}

lsa_status do_scores(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                     const int32_t* row_pos, const void* q_idx, const float* w, float* scores,
                     int64_t ld, void* ws, void* inner_ws, size_t inner_bytes, cudaStream_t s,
                     uint32_t* hist12 = nullptr, bool* hist_done = nullptr, uint32_t* done_ctr = nullptr,
                     bool zeroed = false, bool pdl = false, const ScoresArgs* split = nullptr,
                     int* pool = nullptr) {
  ScoresArgs a = scores_args(d, c, rows, row_seq, row_pos, q_idx, w, scores, ld, ws, inner_ws, inner_bytes);
  if (hist_done) *hist_done = false;
  if (rows == 0 || ld == 0) return LSA_OK;
  if (!force_simt() && scores_tc_supported(a)) {
    a.pdl = pdl;
    if (split) {
      a.grid = split->grid;
      a.split_part = split->split_part;
      a.split_free = split->split_free;
      a.split_busy_us = split->split_busy_us;
      a.split_tile_us = split->split_tile_us;
    }
    if (hist12 && scores_tc_fused_hist_ok(a)) {
      // the scan also counts the first top-k digit; the counters start at
      // zero (cleared here unless the caller already did)
      cudaError_t e = zeroed ? cudaSuccess : cudaMemsetAsync(hist12, 0, topk_hist_zero_bytes(rows), s);
      if (e != cudaSuccess) return LSA_ERR_CUDA;
      a.hist12 = hist12;
      a.done_ctr = done_ctr;  // zeroed with the histograms
      if (hist_done) *hist_done = true;
      if (pool && pool_static_pm() <= 1000 && scores_tc_pool_ok(a)) {  // the pool counter too
        a.pool = pool;
        a.pool_chunk = pool_chunk();
        a.pool_static_pm = pool_static_pm();
      }
    }
    return cuda_status(launch_scores_tc(a, s));
  }
  return cuda_status(launch_scores_simt(a, s));
}

TopkArgs topk_args(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len, int64_t n_cols,
                   int32_t k, int32_t* idx, void* ws, void* inner_ws, bool hist_ready) {
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.rows = rows;
  a.valid_len = valid_len;
  a.n_cols = n_cols;
  a.k = k;
  a.idx = idx;
  a.ws = inner_ws;
  a.status = status_of(ws);
  a.hist_ready = hist_ready;
  return a;
}

lsa_status do_topk(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len, int64_t n_cols,
                   int32_t k, int32_t* idx, void* ws, void* inner_ws, cudaStream_t s, bool hist_ready = false,
                   bool pdl = false, const uint32_t* wait_ctr = nullptr, uint32_t wait_target = 0,
                   bool split_select = false) {
  TopkArgs a = topk_args(scores, ld, rows, valid_len, n_cols, k, idx, ws, inner_ws, hist_ready);
  a.allow_cluster = allow_cluster_topk();
  a.pdl = pdl;
  a.wait_ctr = wait_ctr;
  a.wait_target = wait_target;
  a.split_select = split_select;
  return cuda_status(launch_topk(a, s));
}

AttnArgs attn_args(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq, const void* q,
                   const int32_t* idx, void* out, float* lse, void* ws, void* inner_ws, size_t inner_bytes) {
  AttnArgs a;
  a.cache = view(d, c);
  a.dtype = d->act_dtype;
  a.rows = rows;
  a.row_seq = row_seq;
  a.q = q;
  a.idx = idx;
  a.k = d->top_k;
  a.H = d->n_heads;
  a.D = d->qk_dim;
  a.Dv = d->v_dim;
  a.scale = d->softmax_scale;
  a.out = out;
  a.lse = lse;
  a.ws = inner_ws;
  a.ws_bytes = inner_bytes;
  a.status = status_of(ws);
  return a;
}

lsa_status do_attn(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq, const void* q,
                   const int32_t* idx, void* out, float* lse, void* ws, void* inner_ws, size_t inner_bytes,
                   cudaStream_t s, bool pdl = false, const uint32_t* row_ready = nullptr,
                   const AttnArgs* split = nullptr) {
  AttnArgs a = attn_args(d, c, rows, row_seq, q, idx, out, lse, ws, inner_ws, inner_bytes);
  // in a decode step the kernel before is the step's top-k, which does not write q
  a.pdl = pdl;
  a.q_early = pdl;
  a.row_ready = row_ready;
  if (split) {
    a.split_sel = true;
    a.tk_ws = split->tk_ws;
    a.tk_ncols = split->tk_ncols;
    a.tk_nseg = split->tk_nseg;
    a.tk_seg_len = split->tk_seg_len;
    a.idx_w = split->idx_w;
  }
  if (rows == 0) return LSA_OK;
  if (!force_simt() && attn_tc_supported(a)) return cuda_status(launch_attn_tc(a, s));
  return cuda_status(launch_attn_simt(a, s));
}

}  // namespace
}  // namespace lsa

using namespace lsa;

extern "C" {

size_t lsa_workspace_size(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t op) {
  if (rows < 0 || max_len < 0) return 0;
  switch (op) {
    case LSA_OP_SCORES:
      if (!valid_dims(d)) return 0;
      return kStatusBytes + scores_ws(rows, true);
    case LSA_OP_TOPK:
      if (!d || d->top_k < 1) return 0;
      return topk_call_bytes(rows, max_len, d->top_k);
    case LSA_OP_ATTN:
      if (!valid_dims(d)) return 0;
      return kStatusBytes + attn_ws(d, rows);
    case LSA_OP_DECODE_STEP:
      if (!valid_dims(d)) return 0;
      return step_layout(d, rows, max_len).total;
    case LSA_OP_DECODE_LAYERS:
      if (!valid_dims(d)) return 0;
      return layers_layout(d, rows, max_len).total;
    default:
      return 0;
  }
}

lsa_status lsa_indexer_scores(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                              const int32_t* row_pos, const void* q_idx, const float* w, float* scores,
                              int64_t ld, void* ws, size_t ws_bytes, lsa_stream_t stream) {
  if (!valid_dims(d) || !valid_cache(d, c, true, false)) return LSA_ERR_INVALID_ARG;
  if (rows < 0 || ld < c->max_len) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!q_idx || !w || !scores || !aligned16(q_idx))) return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  if (!row_seq && rows > c->batch) return LSA_ERR_INVALID_ARG;
  const size_t need = kStatusBytes + scores_ws(rows, row_pos != nullptr);
  lsa_status st = ws_check(ws, ws_bytes, need);
  if (st != LSA_OK) return st;
  return do_scores(d, c, rows, row_seq, row_pos, q_idx, w, scores, ld, ws,
                   static_cast<uint8_t*>(ws) + kStatusBytes, ws_bytes - kStatusBytes,
                   reinterpret_cast<cudaStream_t>(stream));
}

lsa_status lsa_topk(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len, int64_t n_cols,
                    int32_t k, int32_t* idx, void* ws, size_t ws_bytes, lsa_stream_t stream) {
  lsa_status st = topk_check_args(scores, ld, rows, n_cols, k, idx);
  if (st != LSA_OK) return st;
  st = ws_check(ws, ws_bytes, topk_call_bytes(rows, n_cols, k));
  if (st != LSA_OK) return st;
  if (rows == 0) return LSA_OK;
  return do_topk(scores, ld, rows, valid_len, n_cols, k, idx, ws, static_cast<uint8_t*>(ws) + kStatusBytes,
                 reinterpret_cast<cudaStream_t>(stream));
}

lsa_status lsa_sparse_attn_decode(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                                  const void* q, const int32_t* idx, void* out, float* lse, void* ws,
                                  size_t ws_bytes, lsa_stream_t stream) {
  if (!valid_dims(d) || !valid_cache(d, c, false, true)) return LSA_ERR_INVALID_ARG;
  if (rows < 0) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!q || !idx || !out || !aligned16(q) || !aligned16(out))) return LSA_ERR_INVALID_ARG;
  if (!row_seq && rows > c->batch) return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  const size_t need = kStatusBytes + attn_ws(d, rows);
  lsa_status st = ws_check(ws, ws_bytes, need);
  if (st != LSA_OK) return st;
  return do_attn(d, c, rows, row_seq, q, idx, out, lse, ws, static_cast<uint8_t*>(ws) + kStatusBytes,
                 ws_bytes - kStatusBytes, reinterpret_cast<cudaStream_t>(stream));
}

static lsa_status decode_step_impl(const lsa_dims* d, const lsa_cache* c, const void* q_idx, const float* w,
                                   const void* q, void* out, float* lse, int32_t* idx_out, int32_t flags, void* ws,
                                   size_t ws_bytes, lsa_stream_t stream, void* const* events) {
  if (!valid_dims(d) || !valid_cache(d, c, true, true)) return LSA_ERR_INVALID_ARG;
  if (flags != LSA_STEP_UNFUSED && flags != LSA_STEP_FUSED) return LSA_ERR_INVALID_ARG;
  const int32_t B = c->batch;
  if (B > 0 && (!q_idx || !w || !q || !out || !aligned16(q_idx) || !aligned16(q) || !aligned16(out)))
    return LSA_ERR_INVALID_ARG;
  if (B > 65535) return LSA_ERR_UNSUPPORTED;
  const StepLayout L = step_layout(d, B, c->max_len);
  lsa_status st = ws_check(ws, ws_bytes, L.total);
  if (st != LSA_OK) return st;
  if (B == 0) return LSA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  auto mark = [&](int i) -> bool {
    if (!events || !events[i]) return true;
    return cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s) == cudaSuccess;
  };
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(base + L.scores_off);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + L.idx_off);
  void* inner = base + L.inner_off;
  const size_t inner_bytes = L.total - L.inner_off;
  const int64_t ld = score_ld(c->max_len);
  // With the tensor-core scan and the three-launch top-k, the scan writes the
  // top-k's first histogram into the top-k workspace (which starts with it).
  if (!mark(0)) return LSA_ERR_CUDA;
  if (flags == LSA_STEP_FUSED && !force_simt()) {
    // one cooperative launch when every stage has its tensor-core / three-pass
    // form and all CTAs fit at once; otherwise the separate launches below
    const ScoresArgs sa = scores_args(d, c, B, nullptr, nullptr, q_idx, w, scores, ld, ws, inner, inner_bytes);
    const TopkArgs ta = topk_args(scores, ld, B, c->seq_lens, c->max_len, d->top_k, idx, ws, inner, true);
    const AttnArgs aa = attn_args(d, c, B, nullptr, q, idx, out, lse, ws, inner, inner_bytes);
    if (step_fused_supported(sa, aa, c->max_len)) {
      const cudaError_t e = launch_step_fused(sa, ta, aa, s);
      if (e == cudaSuccess) {
        for (int i = 1; i < 4; ++i)
          if (!mark(i)) return LSA_ERR_CUDA;
        return LSA_OK;
      }
      if (e != cudaErrorCooperativeLaunchTooLarge) return LSA_ERR_CUDA;
      (void)cudaGetLastError();  // not co-resident on this device: fall back
    }
  }
  uint32_t* hist12 = (!force_simt() && topk_v2_ok(c->max_len)) ? static_cast<uint32_t*>(inner) : nullptr;
  bool hist_done = false;
  // With the histogram built by the scan, the kernels hand over through words
  // zeroed with it: the top-k starts once every scan CTA has counted itself,
  // the attention of a row once that row's selection is written.
  uint32_t *scan_done = nullptr, *sel_done = nullptr;
  int* scan_pool = nullptr;
  if (hist12) topk_step_flags(inner, B, c->max_len, &scan_done, &sel_done, &scan_pool);
  st = do_scores(d, c, B, nullptr, nullptr, q_idx, w, scores, ld, ws, inner, inner_bytes, s, hist12, &hist_done,
                 scan_done, false, false, nullptr, scan_pool);
  if (st != LSA_OK) return st;
  if (!mark(1)) return LSA_ERR_CUDA;
  // The top-k and the attention are launched as programmatic dependents of the
  // kernel before them: their CTAs may be scheduled while it finishes, and
  // they wait for it (griddepcontrol.wait) before reading what it wrote.
  const bool handoff = hist_done && !events;  // events between the kernels would serialise them anyway
  // With the handoffs and the tensor-core attention, the row's last top-k CTA
  // only makes the row's bitmap exact and stores per-segment offsets; each
  // attention CTA compacts its own entries from the segments holding them
  // (and writes them to idx only if the caller asked for the selection).
  // It pays for long rows the one-cluster-per-row top-k cannot take (the
  // full select walks the whole row's bitmap in one CTA: about 27 us at 512K
  // positions, against a few microseconds of compaction per attention CTA);
  // for rows up to about 128K the full select is as fast or faster (measured
  // at 32K and 128K), and rows whose clusters fit take the cluster top-k.
  AttnArgs split;
  bool split_sel = false;
  const bool cluster = allow_cluster_topk() && !force_simt() && topk_cluster_planned(B, c->max_len);
  if (handoff && !cluster && !force_simt() && c->max_len >= split_select_min_cols() &&
      attn_tc_split_fits(B, d->top_k) &&
      attn_tc_supported(attn_args(d, c, B, nullptr, q, idx, out, lse, ws, inner, inner_bytes)) &&
      topk_rows_plan(B, c->max_len, &split.tk_nseg, &split.tk_seg_len)) {
    split_sel = true;
    split.tk_ws = inner;
    split.tk_ncols = c->max_len;
    split.idx_w = idx_out;
  }
  st = do_topk(scores, ld, B, c->seq_lens, c->max_len, d->top_k, idx, ws, inner, s, hist_done, true,
               handoff ? scan_done : nullptr,
               handoff ? static_cast<uint32_t>(scan_tc_grid()) + test_scan_wait_extra() : 0u, split_sel);
  if (st != LSA_OK) return st;
  if (!mark(2)) return LSA_ERR_CUDA;
  st = do_attn(d, c, B, nullptr, q, idx, out, lse, ws, inner, inner_bytes, s, true,
               handoff && !split_sel ? sel_done : nullptr, split_sel ? &split : nullptr);
  if (st != LSA_OK) return st;
  if (!mark(3)) return LSA_ERR_CUDA;
  return LSA_OK;
}

lsa_status lsa_decode_step(const lsa_dims* d, const lsa_cache* c, const void* q_idx, const float* w,
                           const void* q, void* out, float* lse, int32_t* idx_out, int32_t flags, void* ws,
                           size_t ws_bytes, lsa_stream_t stream) {
  return decode_step_impl(d, c, q_idx, w, q, out, lse, idx_out, flags, ws, ws_bytes, stream, nullptr);
}

lsa_status lsa_decode_step_profiled(const lsa_dims* d, const lsa_cache* c, const void* q_idx, const float* w,
                                    const void* q, void* out, float* lse, int32_t* idx_out, int32_t flags,
                                    void* ws, size_t ws_bytes, lsa_stream_t stream, void* const* events) {
  return decode_step_impl(d, c, q_idx, w, q, out, lse, idx_out, flags, ws, ws_bytes, stream, events);
}

lsa_status lsa_decode_layers(const lsa_dims* d, int32_t n_layers, const lsa_cache* caches,
                             const void* const* q_idx, const float* const* w, const void* const* q,
                             void* const* out, float* const* lse, int32_t retention, int32_t route,
                             int32_t* idx_out, void* ws, size_t ws_bytes, lsa_stream_t stream) {
  if (!valid_dims(d) || n_layers < 1 || retention < 1 || !caches || !q || !out) return LSA_ERR_INVALID_ARG;
  if (route != LSA_ROUTE_OWN && route != LSA_ROUTE_PREV) return LSA_ERR_INVALID_ARG;
  const lsa_cache& c0 = caches[0];
  const int32_t B = c0.batch;
  for (int32_t l = 0; l < n_layers; ++l) {
    const lsa_cache& c = caches[l];
    const bool keeps = l % retention == 0;
    if (!valid_cache(d, &c, keeps, true)) return LSA_ERR_INVALID_ARG;
    if (c.batch != B || c.max_len != c0.max_len || c.seq_lens != c0.seq_lens || c.block_table != c0.block_table ||
        c.max_blocks_per_seq != c0.max_blocks_per_seq)
      return LSA_ERR_INVALID_ARG;
    if (B > 0) {
      if (!q[l] || !out[l] || !aligned16(q[l]) || !aligned16(out[l])) return LSA_ERR_INVALID_ARG;
      if (keeps && (!q_idx || !w || !q_idx[l] || !w[l] || !aligned16(q_idx[l]))) return LSA_ERR_INVALID_ARG;
    }
  }
  if (B > 65535) return LSA_ERR_UNSUPPORTED;
  const LayersLayout L = layers_layout(d, B, c0.max_len);
  lsa_status st = ws_check(ws, ws_bytes, L.total);
  if (st != LSA_OK) return st;
  if (B == 0) return LSA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* scores = reinterpret_cast<float*>(base + L.scores_off);
  int32_t* sel[2] = {reinterpret_cast<int32_t*>(base + L.sel_off[0]), reinterpret_cast<int32_t*>(base + L.sel_off[1])};
  void* tk = base + L.tk_off;
  void* at = base + L.at_off;
  const int64_t ld = score_ld(c0.max_len);
  const size_t sel_bytes = static_cast<size_t>(B) * d->top_k * 4;
  int cur = 0;  // the buffer holding the latest indexer layer's selection
  for (int32_t l = 0; l < n_layers; ++l) {
    const lsa_cache* c = &caches[l];
    float* lse_l = lse ? lse[l] : nullptr;
    const int32_t* attended = sel[cur];
    if (l % retention == 0) {
      // MLI: from the second indexer layer on, the attention takes the
      // selection already made and the top-k writes the other buffer
      const bool overlap = route == LSA_ROUTE_PREV && l > 0;
      const int nxt = overlap ? 1 - cur : cur;
      uint32_t* hist12 = (!force_simt() && topk_v2_ok(c->max_len)) ? static_cast<uint32_t*>(tk) : nullptr;
      bool hist_done = false;
      uint32_t *scan_done = nullptr, *sel_done = nullptr;
      int* scan_pool = nullptr;
      if (hist12) topk_step_flags(tk, B, c->max_len, &scan_done, &sel_done, &scan_pool);
      if (overlap) {
        // The attention on the selection already made goes first.  The scan
        // follows as its programmatic dependent (it reads nothing the
        // attention writes) and takes the SMs the attention leaves; the
        // top-k follows the scan.  The counters they share are cleared before
        // the attention, so no copy-engine step separates the kernels.
        const ScoresArgs sa =
            scores_args(d, c, B, nullptr, nullptr, q_idx[l], w[l], scores, ld, ws, tk, L.tk_bytes);
        const bool fused_hist = hist12 && !force_simt() && scores_tc_supported(sa) && scores_tc_fused_hist_ok(sa);
        if (fused_hist && cudaMemsetAsync(hist12, 0, topk_hist_zero_bytes(B), s) != cudaSuccess) return LSA_ERR_CUDA;
        st = do_attn(d, c, B, nullptr, q[l], sel[cur], out[l], lse_l, ws, at, L.at_bytes, s);
        if (st != LSA_OK) return st;
        // The attention's CTAs (one per SM) leave some SMs free: a first scan
        // launch of one CTA per free SM takes the tiles those SMs stream while
        // the attention runs, a second (one CTA per SM) the rest as the
        // attention's CTAs end (each CTA has a static share, so a single
        // launch would end with its last-started CTAs).
        const int sms = scan_tc_grid();
        int cps = 0;
        const bool tc_attn =
            !force_simt() && attn_tc_supported(attn_args(d, c, B, nullptr, q[l], sel[cur], out[l], lse_l, ws, at,
                                                         L.at_bytes));
        const int free_sms = tc_attn ? sms - attn_tc_ctas(B, d->top_k, &cps) : 0;
        uint32_t target = static_cast<uint32_t>(sms);
        if (fused_hist && free_sms > 0) {
          ScoresArgs sp;
          sp.split_free = free_sms;
          sp.split_busy_us = static_cast<float>(kAttnFixedUs + kAttnChunkUs * cps);
          sp.split_tile_us = static_cast<float>(kScanTileUs);
          sp.grid = free_sms;
          sp.split_part = 1;
          st = do_scores(d, c, B, nullptr, nullptr, q_idx[l], w[l], scores, ld, ws, tk, L.tk_bytes, s, hist12,
                         &hist_done, scan_done, true, true, &sp);
          if (st != LSA_OK) return st;
          sp.grid = sms;
          sp.split_part = 2;
          st = do_scores(d, c, B, nullptr, nullptr, q_idx[l], w[l], scores, ld, ws, tk, L.tk_bytes, s, hist12,
                         &hist_done, scan_done, true, true, &sp);
          target = static_cast<uint32_t>(sms + free_sms);
        } else {
          st = do_scores(d, c, B, nullptr, nullptr, q_idx[l], w[l], scores, ld, ws, tk, L.tk_bytes, s,
                         fused_hist ? hist12 : nullptr, &hist_done, scan_done, fused_hist, true);
        }
        if (st != LSA_OK) return st;
        st = do_topk(scores, ld, B, c->seq_lens, c->max_len, d->top_k, sel[nxt], ws, tk, s, hist_done, true,
                     hist_done ? scan_done : nullptr, hist_done ? target : 0u);
      } else {
        st = do_scores(d, c, B, nullptr, nullptr, q_idx[l], w[l], scores, ld, ws, tk, L.tk_bytes, s, hist12,
                       &hist_done, scan_done, false, false, nullptr, scan_pool);
        if (st != LSA_OK) return st;
        st = do_topk(scores, ld, B, c->seq_lens, c->max_len, d->top_k, sel[nxt], ws, tk, s, hist_done, true,
                     hist_done ? scan_done : nullptr, hist_done ? static_cast<uint32_t>(scan_tc_grid()) : 0u);
        if (st != LSA_OK) return st;
        st = do_attn(d, c, B, nullptr, q[l], sel[nxt], out[l], lse_l, ws, at, L.at_bytes, s, true,
                     hist_done ? sel_done : nullptr);
        attended = sel[nxt];
      }
      if (st != LSA_OK) return st;
      cur = nxt;
    } else {
      st = do_attn(d, c, B, nullptr, q[l], attended, out[l], lse_l, ws, at, L.at_bytes, s);
      if (st != LSA_OK) return st;
    }
    if (idx_out && cudaMemcpyAsync(idx_out + static_cast<int64_t>(l) * B * d->top_k, attended, sel_bytes,
                                   cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

lsa_status lsa_candidate_scores(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                                const int32_t* row_pos, const void* q_idx, const float* w, const int32_t* cand,
                                int32_t n_cand, float* scores, int64_t ld, void* ws, size_t ws_bytes,
                                lsa_stream_t stream) {
  if (!valid_dims(d) || !valid_cache(d, c, true, false)) return LSA_ERR_INVALID_ARG;
  if (rows < 0 || n_cand < 0 || ld < n_cand) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!q_idx || !w || !scores || !aligned16(q_idx) || (n_cand > 0 && !cand)))
    return LSA_ERR_INVALID_ARG;
  if (!row_seq && rows > c->batch) return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  lsa_status st = ws_check(ws, ws_bytes, kStatusBytes);
  if (st != LSA_OK) return st;
  if (rows == 0 || ld == 0) return LSA_OK;
  ScoresArgs a = scores_args(d, c, rows, row_seq, row_pos, q_idx, w, scores, ld, ws, nullptr, 0);
  a.cand = cand;
  a.cand_ld = n_cand;
  if (!candidate_scores_tc_supported(a)) return LSA_ERR_UNSUPPORTED;
  return cuda_status(launch_candidate_scores_tc(a, reinterpret_cast<cudaStream_t>(stream)));
}

size_t lsa_two_stage_workspace_size(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t n_cand) {
  if (!valid_dims(d) || rows < 0 || max_len < 0 || n_cand < d->top_k) return 0;
  return two_stage_layout(d, rows, max_len, n_cand).total;
}

lsa_status lsa_two_stage_select(const lsa_dims* d, const lsa_cache* c, const void* compact_keys,
                                const float* compact_scales, int32_t rows, const int32_t* row_seq,
                                const int32_t* row_pos, const void* q_idx, const float* w, int32_t n_cand,
                                int32_t* idx, void* ws, size_t ws_bytes, lsa_stream_t stream) {
  if (!valid_dims(d) || !valid_cache(d, c, true, false)) return LSA_ERR_INVALID_ARG;
  if (rows < 0 || n_cand < d->top_k) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!q_idx || !w || !idx || !aligned16(q_idx) || !compact_keys || !compact_scales ||
                   !aligned16(compact_keys) || !aligned16(compact_scales)))
    return LSA_ERR_INVALID_ARG;
  if (!row_seq && rows > c->batch) return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  if (d->idx_key_dtype != LSA_BF16 || d->act_dtype != LSA_BF16) return LSA_ERR_UNSUPPORTED;
  const TwoStageLayout L = two_stage_layout(d, rows, c->max_len, n_cand);
  lsa_status st = ws_check(ws, ws_bytes, L.total);
  if (st != LSA_OK) return st;
  if (rows == 0) return LSA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* cscores = reinterpret_cast<float*>(base + L.cscores_off);
  int32_t* cand = reinterpret_cast<int32_t*>(base + L.cand_off);
  float* exact = reinterpret_cast<float*>(base + L.exact_off);
  int32_t* slot = reinterpret_cast<int32_t*>(base + L.slot_off);
  void* inner = base + L.inner_off;
  // 1. the compact keys: e4m3 with a per-token scale, the FP8 scan
  lsa_dims d8 = *d;
  d8.idx_key_dtype = LSA_FP8_E4M3;
  lsa_cache c8 = *c;
  c8.idx_keys = compact_keys;
  c8.idx_key_scales = compact_scales;
  ScoresArgs sa = scores_args(&d8, &c8, rows, row_seq, row_pos, q_idx, w, cscores, L.ld_c, ws, inner, L.inner_bytes);
  if (!scores_tc_supported(sa)) return LSA_ERR_UNSUPPORTED;
  st = do_scores(&d8, &c8, rows, row_seq, row_pos, q_idx, w, cscores, L.ld_c, ws, inner, L.inner_bytes, s);
  if (st != LSA_OK) return st;
  // 2. the short list: the n_cand best by compact score (positions past a
  // row's visible range are -inf and never taken)
  const bool by_seq = row_seq == nullptr && row_pos == nullptr;
  st = do_topk(cscores, L.ld_c, rows, by_seq ? c->seq_lens : nullptr, c->max_len, n_cand, cand, ws, inner, s);
  if (st != LSA_OK) return st;
  // 3. the candidates' exact scores from the original keys
  ScoresArgs xa = scores_args(d, c, rows, row_seq, row_pos, q_idx, w, exact, L.ld_x, ws, nullptr, 0);
  xa.cand = cand;
  xa.cand_ld = n_cand;
  if (!candidate_scores_tc_supported(xa)) return LSA_ERR_UNSUPPORTED;
  st = cuda_status(launch_candidate_scores_tc(xa, s));
  if (st != LSA_OK) return st;
  // 4. the k best candidates, ties to the lower entry (= the lower position)
  st = do_topk(exact, L.ld_x, rows, nullptr, n_cand, d->top_k, slot, ws, inner, s);
  if (st != LSA_OK) return st;
  return cuda_status(launch_cand_positions(slot, cand, rows, d->top_k, n_cand, idx, s));
}

size_t lsa_block_select_workspace_size(int32_t rows, int64_t n_cols, int32_t block_size, int32_t n_sel) {
  if (rows < 0 || n_cols < 0 || block_size < 1 || n_sel < 1) return 0;
  const int64_t nb = (n_cols + block_size - 1) / block_size;
  const int64_t nb_ld = score_ld(nb);
  return kStatusBytes + align_up(static_cast<size_t>(rows) * nb_ld * 4) + align_up(topk_ws_bytes(rows, nb, n_sel));
}

lsa_status lsa_block_select(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len, int64_t n_cols,
                            int32_t block_size, int32_t n_sel, int32_t* kept, void* ws, size_t ws_bytes,
                            lsa_stream_t stream) {
  if (rows < 0 || n_cols < 0 || ld < n_cols || block_size < 1 || n_sel < 1) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!scores || !kept)) return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  const int64_t nb = (n_cols + block_size - 1) / block_size;
  const int64_t nb_ld = score_ld(nb);
  lsa_status st = ws_check(ws, ws_bytes, lsa_block_select_workspace_size(rows, n_cols, block_size, n_sel));
  if (st != LSA_OK) return st;
  if (rows == 0) return LSA_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* bscores = reinterpret_cast<float*>(base + kStatusBytes);
  void* inner = base + kStatusBytes + align_up(static_cast<size_t>(rows) * nb_ld * 4);
  if (launch_block_max(scores, ld, rows, valid_len, n_cols, block_size, nb_ld, bscores, s) != cudaSuccess)
    return LSA_ERR_CUDA;
  // every block past a row's visible range scores -inf and is never kept
  return do_topk(bscores, nb_ld, rows, nullptr, nb, n_sel, kept, ws, inner, s);
}

lsa_status lsa_stage_blocks(const lsa_dims* d, const lsa_cache* c, int32_t rows, const int32_t* row_seq,
                            const int32_t* row_pos, const int32_t* kept, int32_t n_sel, int32_t block_size, void* staged_kv,
                            int32_t* staged_table, int32_t* staged_idx, void* ws, size_t ws_bytes,
                            lsa_stream_t stream) {
  if (!valid_dims(d) || !c || !c->seq_lens || c->batch < 0 || c->max_len < 0 || !c->kv) return LSA_ERR_INVALID_ARG;
  if (rows < 0 || n_sel < 1 || block_size < 1) return LSA_ERR_INVALID_ARG;
  if (d->block_size > 0) {  // a kept block of a paged cache is one page
    if (block_size != d->block_size || !c->block_table || c->max_blocks_per_seq < 1 || c->n_blocks < 1)
      return LSA_ERR_INVALID_ARG;
  }
  if (!row_seq && rows > c->batch) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!kept || !staged_kv || !staged_table || !staged_idx || !aligned16(staged_kv)))
    return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  const int64_t row_bytes = static_cast<int64_t>(d->qk_dim) * (d->act_dtype == LSA_F32 ? 4 : 2);
  if (row_bytes % 16) return LSA_ERR_UNSUPPORTED;
  lsa_status st = ws_check(ws, ws_bytes, kStatusBytes);
  if (st != LSA_OK) return st;
  if (rows == 0) return LSA_OK;
  // the source may be host memory the device maps (an offloaded cache): the
  // kernel then reads it through its device address
  CacheView v = view(d, c);
  cudaPointerAttributes pa;
  if (cudaPointerGetAttributes(&pa, c->kv) != cudaSuccess) {
    (void)cudaGetLastError();
    return LSA_ERR_INVALID_ARG;
  }
  if (pa.type == cudaMemoryTypeHost) {
    if (!pa.devicePointer) return LSA_ERR_INVALID_ARG;
    v.kv = pa.devicePointer;
  } else if (pa.type != cudaMemoryTypeDevice && pa.type != cudaMemoryTypeManaged) {
    return LSA_ERR_INVALID_ARG;  // unregistered host memory: the device cannot read it
  }
  if (!aligned16(v.kv)) return LSA_ERR_INVALID_ARG;
  return cuda_status(launch_stage_blocks(v, rows, row_seq, row_pos, kept, n_sel, block_size, row_bytes, staged_kv,
                                         staged_table, staged_idx, status_of(ws),
                                         reinterpret_cast<cudaStream_t>(stream)));
}

size_t lsa_prefill_layers_workspace_size(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t row_block) {
  if (!valid_dims(d) || rows < 0 || max_len < 0 || row_block < 1) return 0;
  return prefill_layout(d, rows, max_len, row_block).total;
}

lsa_status lsa_prefill_layers(const lsa_dims* d, int32_t n_layers, const lsa_cache* caches, int64_t hist_len,
                              const void* const* chunk_kv, int32_t rows, const int32_t* row_pos,
                              const void* const* q_idx, const float* const* w, const void* const* q,
                              void* const* out, float* const* lse, int32_t* const* idx_out, int32_t row_block,
                              void* const* kv_buf, void* ws, size_t ws_bytes, lsa_stream_t compute,
                              lsa_stream_t copy, void* const* events) {
  if (!valid_dims(d) || n_layers < 1 || !caches || rows < 0 || row_block < 1) return LSA_ERR_INVALID_ARG;
  if (d->block_size != 0) return LSA_ERR_INVALID_ARG;  // the streamed history is one contiguous sequence
  const int64_t L = caches[0].max_len;
  if (hist_len < 0 || hist_len > L) return LSA_ERR_INVALID_ARG;
  const int64_t row_bytes = static_cast<int64_t>(d->qk_dim) * (d->act_dtype == LSA_F32 ? 4 : 2);
  for (int32_t l = 0; l < n_layers; ++l) {
    const lsa_cache& c = caches[l];
    if (!valid_cache(d, &c, true, false) || c.batch != 1 || c.max_len != L || !c.kv) return LSA_ERR_INVALID_ARG;
    if (rows > 0) {
      if (!q_idx || !w || !q || !out || !q_idx[l] || !w[l] || !q[l] || !out[l]) return LSA_ERR_INVALID_ARG;
      if (!aligned16(q_idx[l]) || !aligned16(q[l]) || !aligned16(out[l])) return LSA_ERR_INVALID_ARG;
      if (hist_len < L && (!chunk_kv || !chunk_kv[l])) return LSA_ERR_INVALID_ARG;
    }
  }
  if (rows > 0 && (!row_pos || !kv_buf || !kv_buf[0] || !kv_buf[1] || !aligned16(kv_buf[0]) || !aligned16(kv_buf[1]) ||
                   !events || !events[0] || !events[1] || !events[2] || !events[3]))
    return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  const PrefillLayout P = prefill_layout(d, rows, L, row_block);
  lsa_status st = ws_check(ws, ws_bytes, P.total);
  if (st != LSA_OK) return st;
  if (rows == 0) return LSA_OK;
  cudaStream_t sc = reinterpret_cast<cudaStream_t>(compute), sx = reinterpret_cast<cudaStream_t>(copy);
  cudaEvent_t ready[2] = {static_cast<cudaEvent_t>(events[0]), static_cast<cudaEvent_t>(events[1])};
  cudaEvent_t freed[2] = {static_cast<cudaEvent_t>(events[2]), static_cast<cudaEvent_t>(events[3])};
  uint8_t* base = static_cast<uint8_t*>(ws);
  int32_t* row_seq = reinterpret_cast<int32_t*>(base + P.rowseq_off);
  float* scores = reinterpret_cast<float*>(base + P.scores_off);
  int32_t* idx = reinterpret_cast<int32_t*>(base + P.idx_off);
  void* inner = base + P.inner_off;
  if (cudaMemsetAsync(row_seq, 0, static_cast<size_t>(rows) * 4, sc) != cudaSuccess) return LSA_ERR_CUDA;
  const size_t qi_row = static_cast<size_t>(d->n_idx_heads) * d->idx_dim * (d->act_dtype == LSA_F32 ? 4 : 2);
  const size_t q_row = static_cast<size_t>(d->n_heads) * d->qk_dim * (d->act_dtype == LSA_F32 ? 4 : 2);
  const size_t o_row = static_cast<size_t>(d->n_heads) * d->v_dim * (d->act_dtype == LSA_F32 ? 4 : 2);
  for (int32_t l = 0; l < n_layers; ++l) {
    const int b = l & 1;
    // copy side: this layer's history into buffer b once the layer two back
    // has finished reading it, then the chunk's own rows after it
    if (l >= 2 && cudaStreamWaitEvent(sx, freed[b], 0) != cudaSuccess) return LSA_ERR_CUDA;
    uint8_t* buf = static_cast<uint8_t*>(kv_buf[b]);
    if (hist_len > 0 &&
        cudaMemcpyAsync(buf, caches[l].kv, static_cast<size_t>(hist_len * row_bytes), cudaMemcpyDefault, sx) != cudaSuccess)
      return LSA_ERR_CUDA;
    if (hist_len < L && cudaMemcpyAsync(buf + hist_len * row_bytes, chunk_kv[l],
                                        static_cast<size_t>((L - hist_len) * row_bytes), cudaMemcpyDefault,
                                        sx) != cudaSuccess)
      return LSA_ERR_CUDA;
    if (cudaEventRecord(ready[b], sx) != cudaSuccess) return LSA_ERR_CUDA;
    // compute side: the layer's rows, row_block at a time, on buffer b
    if (cudaStreamWaitEvent(sc, ready[b], 0) != cudaSuccess) return LSA_ERR_CUDA;
    lsa_cache cl = caches[l];
    cl.kv = buf;
    for (int32_t r0 = 0; r0 < rows; r0 += row_block) {
      const int32_t nr = rows - r0 < row_block ? rows - r0 : row_block;
      st = do_scores(d, &cl, nr, row_seq, row_pos + r0, static_cast<const uint8_t*>(q_idx[l]) + r0 * qi_row,
                     w[l] + static_cast<int64_t>(r0) * d->n_idx_heads, scores, P.ld, ws, inner, P.inner_bytes, sc);
      if (st != LSA_OK) return st;
      int32_t* sel = idx_out && idx_out[l] ? idx_out[l] + static_cast<int64_t>(r0) * d->top_k : idx;
      st = do_topk(scores, P.ld, nr, nullptr, L, d->top_k, sel, ws, inner, sc);
      if (st != LSA_OK) return st;
      st = do_attn(d, &cl, nr, row_seq, static_cast<const uint8_t*>(q[l]) + r0 * q_row, sel,
                   static_cast<uint8_t*>(out[l]) + r0 * o_row,
                   lse && lse[l] ? lse[l] + static_cast<int64_t>(r0) * d->n_heads : nullptr, ws, inner,
                   P.inner_bytes, sc);
      if (st != LSA_OK) return st;
    }
    if (cudaEventRecord(freed[b], sc) != cudaSuccess) return LSA_ERR_CUDA;
  }
  return LSA_OK;
}

lsa_status lsa_read_device_status(void* ws, int32_t* status, lsa_stream_t stream) {
  if (!ws || !status) return LSA_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  DevStatus h;
  if (cudaMemcpyAsync(&h, ws, sizeof(h), cudaMemcpyDeviceToHost, s) != cudaSuccess) return LSA_ERR_CUDA;
  if (cudaMemsetAsync(ws, 0, sizeof(h), s) != cudaSuccess) return LSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LSA_ERR_CUDA;
  *status = h.code;
  return LSA_OK;
}

lsa_status lsa_get_device_status(void* ws, lsa_stream_t stream) {
  int32_t code = LSA_OK;
  const lsa_status st = lsa_read_device_status(ws, &code, stream);
  return st != LSA_OK ? st : static_cast<lsa_status>(code);
}

int32_t lsa_launch_count(const lsa_dims* d, int32_t rows, int64_t max_len, int32_t op, int32_t causal) {
  if (rows < 0 || max_len < 0) return -1;
  if (op == LSA_OP_TOPK ? (!d || d->top_k < 1) : !valid_dims(d)) return -1;
  if (rows == 0) return 0;
  const bool simt = force_simt();
  int scan = 1;
  int attn = 0;
  bool tc_scan = false;
  if (op != LSA_OP_TOPK) {
    tc_scan = !simt && scores_tc_shape_ok(d->idx_key_dtype, d->act_dtype, d->n_idx_heads, d->idx_dim, d->block_size);
    if (tc_scan) scan = scores_tc_launches(causal != 0);
    if (!simt && attn_tc_shape_ok(d->act_dtype, d->n_heads, d->qk_dim, d->v_dim, d->block_size))
      attn = attn_tc_launches(rows, d->n_heads, d->top_k);
    else
      attn = attn_simt_launches(rows, d->n_heads, d->top_k);
  }
  switch (op) {
    case LSA_OP_SCORES: return scan;
    case LSA_OP_TOPK: return topk_launches(max_len);
    case LSA_OP_ATTN: return attn;
    case LSA_OP_DECODE_STEP: {
      // the tensor-core scan of a decode step also builds the top-k's first histogram
      const int topk = topk_launches(max_len) - (tc_scan && causal == 0 && topk_v2_ok(max_len) ? 1 : 0);
      return scan + topk + attn;
    }
    case LSA_OP_DECODE_STEP_FUSED: {
      const bool fused = !simt && causal == 0 && topk_v2_ok(max_len) &&
                         scores_tc_shape_ok(d->idx_key_dtype, d->act_dtype, d->n_idx_heads, d->idx_dim,
                                            d->block_size) &&
                         attn_tc_shape_ok(d->act_dtype, d->n_heads, d->qk_dim, d->v_dim, d->block_size);
      const int topk = topk_launches(max_len) - (tc_scan && causal == 0 && topk_v2_ok(max_len) ? 1 : 0);
      return fused ? 1 : scan + topk + attn;
    }
    default: return -1;
  }
}

const char* lsa_status_string(lsa_status s) {
  switch (s) {
    case LSA_OK: return "ok";
    case LSA_ERR_INVALID_ARG: return "invalid argument";
    case LSA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case LSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case LSA_ERR_CUDA: return "CUDA runtime error";
    case LSA_ERR_TIMEOUT: return "device wait timed out";
    case LSA_ERR_BOUNDS: return "device index out of bounds";
    default: return "unknown status";
  }
}

int32_t lsa_version(void) { return LSA_VERSION; }

#ifdef LSA_TEST_HOOKS
lsa_status lsa_test_set_hooks(int32_t force_simt_path, int64_t split_select_min_cols_, uint32_t scan_wait_extra,
                              int32_t no_cluster_topk) {
  g_hooks.no_cluster_topk = no_cluster_topk != 0;
  g_hooks.force_simt = force_simt_path != 0;
  g_hooks.split_select_min_cols = split_select_min_cols_ < 0 ? kSplitSelectMinCols : split_select_min_cols_;
  g_hooks.scan_wait_extra = scan_wait_extra;
  return LSA_OK;
}

lsa_status lsa_test_set_scan_pool(int32_t static_pm, int32_t chunk) {
  g_hooks.pool_static_pm = static_pm < 0 ? kPoolStaticPm : static_pm;
  g_hooks.pool_chunk = chunk <= 0 ? kPoolChunk : chunk;
  return LSA_OK;
}
#endif

}  // extern "C"
