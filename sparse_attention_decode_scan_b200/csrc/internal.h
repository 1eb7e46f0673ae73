// Internal launch interface between the C-ABI layer (abi.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lsa.h"

namespace lsa {

struct DevStatus;

// Planning constant: B200 has 148 SMs.  Workspace sizes depend on launch plans,
// so plans use this fixed count (not a device query) to stay host-computable.
constexpr int kPlanSMs = 148;

struct CacheView {
  const void* idx_keys;
  const float* idx_key_scales;
  const void* kv;
  const int32_t* block_table;
  int32_t max_blocks;
  int64_t n_blocks;
  int64_t max_len;
  const int32_t* seq_lens;
  int32_t batch;
  int32_t block_size;
};

struct ScoresArgs {
  CacheView cache;
  int32_t key_dtype, q_dtype;
  int32_t H, dI;
  int32_t rows;
  const int32_t* row_seq;
  const int32_t* row_pos;
  const void* q_idx;
  const float* w;
  float* scores;
  int64_t ld;
  DevStatus* status;
  void* plan_ws;       // tensor-core path scratch (row groups), may be null
  size_t plan_bytes;
  uint32_t* hist12;    // if set: per-row histogram of score-key bits [31:20] ([rows][4096],
                       // zeroed by the caller), accumulated by the scan for the top-k
  uint32_t* done_ctr = nullptr;  // if set (zeroed by the caller): every CTA adds 1 once its
                                 // scores and histogram counts are written and fenced
  // Candidate re-scoring (the second stage of the two-stage search): if set,
  // row r scores only the positions cand[r * cand_ld + j], j < cand_ld
  // (ascending, -1 = no candidate), and scores[r][j] is the score of entry j
  // (-inf for -1; NaN and LSA_ERR_BOUNDS for a position outside the row's
  // visible range or a bad block).  bf16 keys only.
  const int32_t* cand = nullptr;
  int32_t cand_ld = 0;
  // Tensor-core scan launched as a programmatic dependent of the kernel before
  // it, which writes nothing the scan reads (the scan never waits for it).
  bool pdl = false;
  // Tensor-core scan: `grid` CTAs (0: one per SM).  split_part 1 or 2: the
  // launch covers the first or the second part of the rows' tiles, the first
  // being what split_free CTAs stream in split_busy_us while the other SMs
  // are held by another kernel (one tile per split_tile_us); 0: every tile.
  int grid = 0;
  int split_part = 0;
  int split_free = 0;
  float split_busy_us = 0.f, split_tile_us = 1.f;
  // Tensor-core decode scan (one query row per tile, rows <= 256): if set
  // (zeroed by the caller), the CTAs share the first pool_static_pm
  // thousandths of the tiles evenly and claim the rest from this counter in
  // chunks of pool_chunk tiles (a dynamic tail; off unless a test asks).
  int* pool = nullptr;
  int pool_chunk = 0;
  int pool_static_pm = 1000;
};

// ---- indexer
cudaError_t launch_scores_simt(const ScoresArgs& a, cudaStream_t s);
// shape/dtype test of the tensor-core scan (alignment is checked separately)
bool scores_tc_shape_ok(int32_t key_dtype, int32_t q_dtype, int32_t H, int32_t dI, int32_t block_size);
int scores_tc_launches(bool causal);
bool scores_tc_supported(const ScoresArgs& a);
// the pooled tile schedule applies: one query row per tile, rows <= 256
bool scores_tc_pool_ok(const ScoresArgs& a);
size_t scores_tc_ws_bytes(int32_t rows, bool causal);
cudaError_t launch_scores_tc(const ScoresArgs& a, cudaStream_t s);
// Candidate re-scoring on the tensor cores (a.cand set): shape and alignment
// test, and the launch.
bool candidate_scores_tc_supported(const ScoresArgs& a);
cudaError_t launch_candidate_scores_tc(const ScoresArgs& a, cudaStream_t s);
// Block selection (blocks.cu): block scores [rows, nb_ld] = the largest visible
// token score per block; the kept blocks' KV rows copied into a staging pool
// (staged block r * n_sel + i), its block table and the staged positions.
cudaError_t launch_block_max(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len, int64_t n_cols,
                             int32_t block_size, int64_t nb_ld, float* out, cudaStream_t s);
cudaError_t launch_stage_blocks(const CacheView& c, int32_t rows, const int32_t* row_seq, const int32_t* row_pos,
                                const int32_t* kept, int32_t n_sel, int32_t sel_bs, int64_t row_bytes, void* staged,
                                int32_t* staged_table, int32_t* staged_idx, DevStatus* status, cudaStream_t s);
// idx[r][j] = cand[r][slot[r][j]] (-1 for slot -1): candidate entries -> positions.
cudaError_t launch_cand_positions(const int32_t* slot, const int32_t* cand, int32_t rows, int32_t k, int32_t n_cand,
                                  int32_t* idx, cudaStream_t s);

// ---- top-k
struct TopkPlan {
  int32_t nseg;
  int64_t seg_len;
};
TopkPlan topk_plan(int32_t rows, int64_t n_cols);
size_t topk_ws_bytes(int32_t rows, int64_t n_cols, int32_t k);
// Argument checks of the top-k entry points (lsa_topk, lsa_topk_noalloc), and
// the bytes either needs: status word plus the 256-aligned top-k scratch.
lsa_status topk_check_args(const float* scores, int64_t ld, int32_t rows, int64_t n_cols, int32_t k,
                           const int32_t* idx);
size_t topk_call_bytes(int32_t rows, int64_t n_cols, int32_t k);
int topk_launches(int64_t n_cols);

struct TopkArgs {
  const float* scores;
  int64_t ld;
  int32_t rows;
  const int32_t* valid_len;
  int64_t n_cols;
  int32_t k;
  int32_t* idx;
  void* ws;            // topk_ws_bytes bytes (256-aligned)
  DevStatus* status;
  bool hist_ready;     // the first histogram and list counters are already in ws
  bool pdl = false;    // launched as a programmatic dependent of the kernel before it (decode step)
  // Decode step: instead of waiting for the scan grid to complete, wait until
  // *wait_ctr reaches wait_target (the scan's CTAs, each after its writes);
  // each row's selection then raises its flag in the layout's sel_done.
  const uint32_t* wait_ctr = nullptr;
  uint32_t wait_target = 0;
  // Decode step: the row's last collect CTA runs the split select (exact
  // bitmap and per-segment offsets, flag selready = 1) instead of writing idx
  // (or, when the split select cannot, the full select, flag 2).
  bool split_select = false;
  // rows up to tk::kClMaxCols take the one-cluster-per-row kernel (the test
  // build can turn it off to compare the two paths)
  bool allow_cluster = true;
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);
// The decode step's handoff words inside the top-k workspace (zeroed with its
// head): the count of finished scan CTAs, the per-row selection flags and the
// scan's tile pool counter.
void topk_step_flags(void* ws, int32_t rows, int64_t n_cols, uint32_t** scan_done, uint32_t** sel_done,
                     int** scan_pool = nullptr);
// Collect segments per row and their length of the one-launch top-k for these
// sizes; false on a CUDA error.
bool topk_rows_plan(int32_t rows, int64_t n_cols, int* nseg, int64_t* seg_len);
// The three-launch top-k applies (rows up to 2^19 entries); its first
// histogram then sits at the start of the top-k workspace, followed by the
// list counters; topk_hist_zero_bytes of them must be zero before the scan.
bool topk_v2_ok(int64_t n_cols);
// Rows this short may take the one-cluster-per-row top-k.
bool topk_cluster_ok(int64_t n_cols);
// True if these rows take the one-cluster-per-row top-k (their clusters fit
// on the device at once); a decode step then skips the split select.
bool topk_cluster_planned(int32_t rows, int64_t n_cols);
size_t topk_hist_zero_bytes(int32_t rows);
// true if the scan can accumulate the top-k histogram itself
bool scores_tc_fused_hist_ok(const ScoresArgs& a);
// segments of the top-k collect pass, about target_ctas CTAs in total
TopkPlan topk_collect_plan(int32_t rows, int64_t n_cols, int32_t target_ctas);
// tensor maps of the tensor-core scan (keys; FP8 scales)
cudaError_t scan_tc_maps(const ScoresArgs& a, CUtensorMap* tmap, CUtensorMap* smap);
// CTAs of a tensor-core scan launch (one per SM).
int scan_tc_grid();

// ---- sparse attention
struct AttnArgs {
  CacheView cache;
  int32_t dtype;
  int32_t rows;
  const int32_t* row_seq;
  const void* q;
  const int32_t* idx;
  int32_t k;
  int32_t H, D, Dv;
  float scale;
  void* out;
  float* lse;
  void* ws;
  size_t ws_bytes;
  DevStatus* status;
  bool pdl = false;      // launched as a programmatic dependent of the kernel before it (decode step)
  bool q_early = false;  // with pdl: q may be read before the kernel before it completes
  // Decode step: the selection of row r may be read once row_ready[r] != 0
  // (raised by the top-k after writing it); null: wait for the kernel before.
  const uint32_t* row_ready = nullptr;
  // Decode step with the top-k's split select: each CTA compacts its split's
  // entries from the exact bitmap itself (top-k workspace tk_ws, n_cols score
  // columns per row in tk_nseg segments of tk_seg_len); idx_w (or null):
  // where CTAs of the first head half store them.
  bool split_sel = false;
  void* tk_ws = nullptr;
  int64_t tk_ncols = 0;
  int tk_nseg = 0;
  int64_t tk_seg_len = 0;
  int32_t* idx_w = nullptr;
};
size_t attn_simt_ws_bytes(int32_t rows, int32_t H, int32_t Dv, int32_t k);
cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s);
int attn_simt_launches(int32_t rows, int32_t H, int32_t k);
bool attn_tc_shape_ok(int32_t dtype, int32_t H, int32_t D, int32_t Dv, int32_t block_size);
int attn_tc_launches(int32_t rows, int32_t H, int32_t k);
bool attn_tc_supported(const AttnArgs& a);
// Whether each split of the tensor-core attention holds at most one row table
// of entries (needed for it to compact its entries itself).
bool attn_tc_split_fits(int32_t rows, int32_t k);
// CTAs of the tensor-core attention's launch for `rows` rows and k entries
// (and the 64-entry chunks each CTA works through).
int attn_tc_ctas(int32_t rows, int32_t k, int* chunks_per_cta);
size_t attn_tc_ws_bytes(int32_t rows, int32_t H, int32_t D, int32_t Dv, int32_t k);
cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s);
// exact merge of per-split softmax partials (shared by both attention paths)
cudaError_t launch_lse_merge(const AttnArgs& a, int nsplit, const float* part_o, const float* part_lse,
                             cudaStream_t s);

// ---- fused decode step: scan -> top-k -> attention in one cooperative launch
// (one CTA per SM, grid-wide barriers between the phases).  Applies when the
// tensor-core scan with its histogram, the three-launch top-k and the
// tensor-core attention all apply.  Workspace: the top-k workspace `topk.ws`,
// of step_fused_ws_bytes bytes.
bool step_fused_supported(const ScoresArgs& sa, const AttnArgs& aa, int64_t n_cols);
size_t step_fused_ws_bytes(int32_t rows, int64_t n_cols, int32_t k);
cudaError_t launch_step_fused(const ScoresArgs& sa, const TopkArgs& ta, const AttnArgs& aa, cudaStream_t s);

}  // namespace lsa
