// Sparse MQA decode on the sm_100a tensor cores: the standalone kernel (one CTA
// per (split, 64 heads, row) around the CTA body of attn_tc.cuh) and its host
// side (split plan, workspace, launch).
#include <math.h>

#include "common.cuh"
#include "host_util.h"
#include "internal.h"
#include "tc.cuh"

#include <string.h>

#include "attn_tc.cuh"

namespace lsa {
namespace {

using namespace attn;

__global__ void __launch_bounds__(kThreads, 1) k_attn_tc(const TcAttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  // a programmatic dependent (the layer's scan under the MLI route, which
  // reads nothing this kernel writes) may take the SMs this grid leaves free
  tc::griddep_launch_dependents();
  if ((threadIdx.x >> 5) == kWarpMma) {
    tc::tmem_alloc(&tmem_slot, kTmemCols);
    tc::tc_fence_before();
  }
  attn_cta(P, smem_raw, blockIdx.x, blockIdx.y, blockIdx.z, &tmem_slot);
  if ((threadIdx.x >> 5) == kWarpMma) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_slot, kTmemCols);
  }
}


inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Clusters of `n` attention CTAs the current device keeps resident at once
// (queried once per device and n, under a lock; 0 when clusters of that size
// are refused).  The cluster merge is used only when all of a launch's
// clusters fit in one wave, as the split plan assumes.
int resident_clusters(int n) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static int cached[kMaxDev][17];
  static bool init = false;
  if (n < 2 || n > 16) return 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) {
    (void)cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!init) {
    for (auto& row : cached)
      for (int& v : row) v = -1;
    init = true;
  }
  if (cached[dev][n] >= 0) return cached[dev][n];
  cached[dev][n] = 0;
  if (ensure_dyn_smem(k_attn_tc, kSmemBytes) != cudaSuccess ||
      (n > 8 && cudaFuncSetAttribute(k_attn_tc, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess)) {
    (void)cudaGetLastError();
    return 0;
  }
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(n), 1, 1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = static_cast<unsigned>(n);
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int c = 0;
  if (cudaOccupancyMaxActiveClusters(&c, k_attn_tc, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    c = 0;
  }
  cached[dev][n] = c;
  return c;
}

size_t align256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace

bool attn_tc_shape_ok(int32_t dtype, int32_t H, int32_t D, int32_t Dv, int32_t) {
  return dtype == LSA_BF16 && H == kHeadsAll && D == kD && Dv == kDv;
}

int attn_tc_launches(int32_t, int32_t, int32_t) { return 1; }

int attn_tc_ctas(int32_t rows, int32_t k, int* chunks_per_cta) {
  const int ns = tc_nsplit(rows, k);
  const int chunks = (k + kChunk - 1) / kChunk;
  if (chunks_per_cta) *chunks_per_cta = (chunks + ns - 1) / ns;
  return ns * 2 * rows;
}

bool attn_tc_split_fits(int32_t rows, int32_t k) {
  const int ns = tc_nsplit(rows, k);
  const int chunks = (k + kChunk - 1) / kChunk;
  return ((chunks + ns - 1) / ns) * kChunk <= kRowTab;
}

bool attn_tc_supported(const AttnArgs& a) {
  // KV rows are kept as 32-bit indices
  const int64_t kv_rows = a.cache.block_size > 0 ? a.cache.n_blocks * a.cache.block_size
                                                 : static_cast<int64_t>(a.cache.batch) * a.cache.max_len;
  return attn_tc_shape_ok(a.dtype, a.H, a.D, a.Dv, a.cache.block_size) && aligned16(a.cache.kv) && aligned16(a.q) &&
         aligned16(a.out) && kv_rows < (1LL << 31);
}

size_t attn_tc_ws_bytes(int32_t rows, int32_t H, int32_t D, int32_t Dv, int32_t k) {
  if (H != kHeadsAll || D != kD || Dv != kDv) return 0;
  const int ns = tc_nsplit(rows, k);
  if (ns == 1) return 0;
  return align256(static_cast<size_t>(rows) * 2 * sizeof(int)) +
         align256(static_cast<size_t>(rows) * ns * H * sizeof(float)) +
         align256(static_cast<size_t>(rows) * ns * H * Dv * sizeof(float));
}

cudaError_t launch_attn_tc(const AttnArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  TcAttnParams P;
  P.a = a;
  P.nsplit = tc_nsplit(a.rows, a.k);
  const int chunks = (a.k + kChunk - 1) / kChunk;
  P.split_len = ((chunks + P.nsplit - 1) / P.nsplit) * kChunk;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
  const size_t cnt_b = align256(static_cast<size_t>(a.rows) * 2 * sizeof(int));
  const size_t lse_b = align256(static_cast<size_t>(a.rows) * P.nsplit * kHeadsAll * sizeof(float));
  P.counters = reinterpret_cast<int*>(ws);
  P.part_lse = reinterpret_cast<float*>(ws + cnt_b);
  P.part_o = reinterpret_cast<float*>(ws + cnt_b + lse_b);
  {
    cudaError_t e = ensure_dyn_smem(k_attn_tc, kSmemBytes);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(P.nsplit, 2, a.rows);
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = kSmemBytes;
  cfg.stream = s;
  cudaLaunchAttribute attr_c[2];
  attr_c[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr_c[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr_c;
  if (P.nsplit == 1) {
    P.merge = kMergeSeparate;  // nothing to merge
    cfg.attrs = attr_c + 1;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_attn_tc, P);
  }
  cfg.numAttrs = 1;
  // The split CTAs of a (row, half) as one thread-block cluster merge through
  // distributed shared memory; the hardware schedules a cluster's CTAs
  // together, so no counters, global partials or cooperative launch are needed.
  if (resident_clusters(P.nsplit) >= 2 * a.rows) {
    P.merge = kMergeCluster;
    attr_c[0].id = cudaLaunchAttributeClusterDimension;
    attr_c[0].val.clusterDim.x = static_cast<unsigned>(P.nsplit);
    attr_c[0].val.clusterDim.y = 1;
    attr_c[0].val.clusterDim.z = 1;
    cfg.numAttrs = a.pdl ? 2 : 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, k_attn_tc, P);
    cfg.numAttrs = 1;
    if (e == cudaSuccess) return cudaSuccess;
    (void)cudaGetLastError();  // refused: the merge below
  }
  cudaError_t e = cudaMemsetAsync(P.counters, 0, static_cast<size_t>(a.rows) * 2 * sizeof(int), s);
  if (e != cudaSuccess) return e;
  // The split CTAs of a row meet in the kernel, which needs them all resident:
  // a cooperative launch guarantees that or refuses.  Refused (fewer SMs than
  // the one-wave plan assumes), the partials are merged by a second launch.
  P.merge = kMergeInKernel;
  attr_c[0].id = cudaLaunchAttributeCooperative;
  attr_c[0].val.cooperative = 1;
  e = cudaLaunchKernelEx(&cfg, k_attn_tc, P);
  if (e == cudaSuccess) return cudaSuccess;
  if (e != cudaErrorCooperativeLaunchTooLarge) return e;
  (void)cudaGetLastError();
  P.merge = kMergeSeparate;
  k_attn_tc<<<grid, kThreads, kSmemBytes, s>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_lse_merge(a, P.nsplit, P.part_o, P.part_lse, s);
}

}  // namespace lsa
