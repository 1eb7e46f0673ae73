// Block-level selection with a staged copy of the kept blocks (the SparDA
// abstract, page 4 of the sources: the selector picks the KV blocks a layer
// needs, and a forecast of the next layer's blocks lets their host-to-device
// copy overlap the current layer).  Kernels:
//   k_block_max     the score of every block of block_size positions: the
//                   largest token score among its visible positions;
//   k_stage_blocks  copies each row's kept blocks (through the cache's block
//                   table) into a staging pool, and writes the staged block
//                   table and the positions the attention then reads.
// The kept blocks themselves come from the top-k kernels run over the block
// scores.  The source cache may be in host memory the device can map (an
// offloaded KV cache); the copy then reads it over the host link.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kBT = 256;

// One thread per block: the largest of the block's visible scores (-inf if
// none; NaN entries are skipped, as the top-k never takes them).
__global__ void __launch_bounds__(kBT) k_block_max(const float* __restrict__ scores, int64_t ld, int32_t rows,
                                                   const int32_t* __restrict__ valid_len, int64_t n_cols,
                                                   int32_t block_size, int64_t nb_ld, float* __restrict__ out) {
  const int r = blockIdx.y;
  const int64_t blk = blockIdx.x * static_cast<int64_t>(kBT) + threadIdx.x;
  const int64_t nb = (n_cols + block_size - 1) / block_size;
  if (blk >= nb_ld) return;
  float* o = out + static_cast<int64_t>(r) * nb_ld;
  if (blk >= nb) {
    o[blk] = -INFINITY;
    return;
  }
  int64_t n = n_cols;
  if (valid_len) {
    const int64_t v = __ldg(valid_len + r);
    n = v < 0 ? 0 : (v < n ? v : n);
  }
  const int64_t p0 = blk * block_size;
  const int64_t p1 = p0 + block_size < n ? p0 + block_size : n;
  const float* row = scores + static_cast<int64_t>(r) * ld;
  float m = -INFINITY;
  for (int64_t p = p0; p < p1; ++p) {
    const float x = __ldg(row + p);
    m = x > m ? x : m;  // NaN compares false: skipped
  }
  o[blk] = m;
}

// CTA (i, r): kept block i of row r (a block is sel_bs consecutive positions;
// in a paged cache it must be one page).  Copies the block's KV rows from the
// source cache into staged block r * n_sel + i (rows past the sequence are
// zero-filled), and writes the staged table entry and the block's positions in
// the staged sequence (i * sel_bs + t, or -1 where the source position is past
// the sequence or no block was kept).
__global__ void __launch_bounds__(kBT) k_stage_blocks(CacheView c, int32_t rows, const int32_t* __restrict__ row_seq,
                                                      const int32_t* __restrict__ row_pos,
                                                      const int32_t* __restrict__ kept, int32_t n_sel, int32_t sel_bs,
                                                      int64_t row_bytes, uint8_t* __restrict__ staged,
                                                      int32_t* __restrict__ staged_table,
                                                      int32_t* __restrict__ staged_idx, DevStatus* status) {
  const int i = blockIdx.x, r = blockIdx.y;
  const int b = row_seq ? __ldg(row_seq + r) : r;
  const bool ok = b >= 0 && b < c.batch;
  int64_t L = ok ? __ldg(c.seq_lens + b) : 0;
  L = L < 0 ? 0 : (L > c.max_len ? c.max_len : L);
  if (row_pos) {  // causal row: positions up to its own
    const int64_t p = static_cast<int64_t>(__ldg(row_pos + r)) + 1;
    L = p < L ? (p < 0 ? 0 : p) : L;
  }
  const int32_t blk = __ldg(kept + static_cast<int64_t>(r) * n_sel + i);
  // first source row of the block (-1: none kept, or out of range)
  int64_t src_row0 = -1;
  if (ok && blk >= 0 && static_cast<int64_t>(blk) * sel_bs < L) {
    if (c.block_size > 0) {
      if (blk < c.max_blocks) {
        const int32_t pb = __ldg(c.block_table + static_cast<int64_t>(b) * c.max_blocks + blk);
        if (pb >= 0 && pb < c.n_blocks) src_row0 = static_cast<int64_t>(pb) * c.block_size;
      }
    } else {
      src_row0 = static_cast<int64_t>(b) * c.max_len + static_cast<int64_t>(blk) * sel_bs;
    }
    if (src_row0 < 0 && threadIdx.x == 0) record_error(status, LSA_ERR_BOUNDS, r, blk);
  }
  const int64_t dst_blk = static_cast<int64_t>(r) * n_sel + i;
  if (threadIdx.x == 0) staged_table[dst_blk] = src_row0 >= 0 ? static_cast<int32_t>(dst_blk) : -1;
  const int64_t pos0 = static_cast<int64_t>(blk) * sel_bs;
  for (int t = threadIdx.x; t < sel_bs; t += kBT)
    staged_idx[static_cast<int64_t>(r) * n_sel * sel_bs + static_cast<int64_t>(i) * sel_bs + t] =
        (src_row0 >= 0 && pos0 + t < L) ? i * sel_bs + t : -1;
  if (src_row0 < 0) return;
  const int64_t per_row = row_bytes / 16;
  const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(c.kv) + src_row0 * row_bytes);
  uint4* dst = reinterpret_cast<uint4*>(staged + dst_blk * sel_bs * row_bytes);
  const int64_t n16 = sel_bs * per_row;
  const int64_t live16 = (L - pos0 < sel_bs ? L - pos0 : sel_bs) * per_row;  // rows inside the sequence
  // eight 16-byte loads in flight per thread (the source may sit across the host link)
  for (int64_t k0 = threadIdx.x; k0 < n16; k0 += 8 * kBT) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = k0 + u * kBT < live16 ? src[k0 + u * kBT] : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (k0 + u * kBT < n16) dst[k0 + u * kBT] = v[u];
  }
}

}  // namespace

cudaError_t launch_block_max(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len, int64_t n_cols,
                             int32_t block_size, int64_t nb_ld, float* out, cudaStream_t s) {
  if (rows == 0 || nb_ld == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((nb_ld + kBT - 1) / kBT), static_cast<unsigned>(rows));
  k_block_max<<<grid, kBT, 0, s>>>(scores, ld, rows, valid_len, n_cols, block_size, nb_ld, out);
  return cudaGetLastError();
}

cudaError_t launch_stage_blocks(const CacheView& c, int32_t rows, const int32_t* row_seq, const int32_t* row_pos,
                                const int32_t* kept, int32_t n_sel, int32_t sel_bs, int64_t row_bytes, void* staged,
                                int32_t* staged_table, int32_t* staged_idx, DevStatus* status, cudaStream_t s) {
  if (rows == 0 || n_sel == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>(n_sel), static_cast<unsigned>(rows));
  k_stage_blocks<<<grid, kBT, 0, s>>>(c, rows, row_seq, row_pos, kept, n_sel, sel_bs, row_bytes, static_cast<uint8_t*>(staged),
                                      staged_table, staged_idx, status);
  return cudaGetLastError();
}

}  // namespace lsa
