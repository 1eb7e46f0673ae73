// Last step of the two-stage indexer search (LeanSparse episode page, summary:
// search compact keys, fetch a short list of the originals, rank them
// exactly): the top-k over the candidates' exact scores names candidate
// entries; this kernel turns them into cache positions.
#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.h"

namespace lsa {
namespace {

// idx[r][j] = cand[r][slot[r][j]] (or -1 where slot is -1).  The slots come
// ascending from the top-k and the candidate list is ascending in position,
// so each output row stays ascending.
__global__ void k_cand_positions(const int32_t* __restrict__ slot, const int32_t* __restrict__ cand, int32_t rows,
                                 int32_t k, int32_t n_cand, int32_t* __restrict__ idx) {
  const int64_t n = static_cast<int64_t>(rows) * k;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t r = i / k;
    const int32_t sl = slot[i];
    idx[i] = (sl >= 0 && sl < n_cand) ? cand[r * n_cand + sl] : -1;
  }
}

}  // namespace

cudaError_t launch_cand_positions(const int32_t* slot, const int32_t* cand, int32_t rows, int32_t k, int32_t n_cand,
                                  int32_t* idx, cudaStream_t s) {
  const int64_t n = static_cast<int64_t>(rows) * k;
  if (n == 0) return cudaSuccess;
  int64_t blocks = (n + 255) / 256;
  if (blocks > 4 * kPlanSMs) blocks = 4 * kPlanSMs;
  k_cand_positions<<<static_cast<unsigned>(blocks), 256, 0, s>>>(slot, cand, rows, k, n_cand, idx);
  return cudaGetLastError();
}

}  // namespace lsa
