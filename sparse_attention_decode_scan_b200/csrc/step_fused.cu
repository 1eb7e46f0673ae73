// Fused decode step: the lightning-indexer scan, the top-k and the sparse
// attention of one decode step in a single cooperative launch of one CTA per SM
// (the optional fused decode kernel the MLI page mentions for DeepSeek-V3.2,
// built here for sm_100a).
//
// Phases, separated by grid-wide barriers with bounded waits:
//   1. scan (threads 0-223): the tensor-core scan of every row, which also
//      builds each row's first top-k digit histogram;
//   2. top-k collect (threads 0-255): bitmap words and threshold-bin
//      candidates, segments of every row over all CTAs;
//   3. top-k select (threads 0-255): one row per CTA;
//   4. attention (all 288 threads): the (split, 64 heads, row) CTAs with their
//      last-CTA log-sum-exp merge.
// Each phase runs the CTA bodies of the standalone kernels, so the step's
// results are those of the separate launches.  The TMEM columns are allocated
// once for the whole launch.  Data a phase reads that an earlier phase wrote
// (scores, histograms, selections) is read through L2 (ld.cg), never through
// the non-coherent read-only path.
#include <cuda.h>
#include <string.h>

#include "attn_tc.cuh"
#include "common.cuh"
#include "host_util.h"
#include "internal.h"
#include "scan_tc.cuh"
#include "tc.cuh"
#include "topk_sel.cuh"

namespace lsa {
namespace {

constexpr int kFusedThreads = attn::kThreads;  // 288
constexpr int kSelThreads = 256;               // threads of the top-k phases
constexpr uint32_t kFusedTmemCols = 512;       // the attention's columns; the scan uses the first 128 or 256
constexpr int kWarpTmem = 1;                   // allocates and frees the TMEM columns (the scan's MMA warp)
static_assert(scan::kThreads <= kFusedThreads && tk::kCollectThreads <= kFusedThreads && kSelThreads <= kFusedThreads,
              "phase thread counts");
static_assert(scan::kWarpMma == kWarpTmem, "the scan's MMA warp owns the TMEM allocation");

struct FusedParams {
  ScoresArgs scan;
  TopkArgs topk;
  attn::TcAttnParams attn;
  int32_t collect_nseg;
  int64_t collect_seg_len;
  uint32_t* bar;  // grid-barrier arrivals (zeroed before the launch)
};

// All CTAs arrive, then wait (bounded) until gridDim.x * phase arrivals are
// counted.  Returns false after a timeout (recorded as LSA_ERR_TIMEOUT), after
// which the caller skips the remaining phases.
__device__ bool grid_sync(uint32_t* bar, uint32_t phase, DevStatus* status, volatile int* s_ok) {
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(bar, 1u);
    const uint32_t target = gridDim.x * phase;
    int ok = 1;
    const uint64_t t0 = tc::globaltimer_ns();
    for (;;) {
      uint32_t v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
      if (v >= target) break;
      if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) {
        ok = 0;
        record_error(status, LSA_ERR_TIMEOUT, -1, static_cast<int>(phase));
        break;
      }
      __nanosleep(64);
    }
    __threadfence();
    *s_ok = ok;
  }
  __syncthreads();
  return *s_ok != 0;
}

constexpr size_t kScratchBytes = (sizeof(tk::TkScratch) + 255) / 256 * 256;

template <int KDT>
__global__ void __launch_bounds__(kFusedThreads, 1) k_step_fused(const __grid_constant__ CUtensorMap tmap,
                                                                  const __grid_constant__ CUtensorMap smap,
                                                                  const FusedParams F) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  __shared__ int s_ok;
  const int warp = threadIdx.x >> 5;
  if (warp == kWarpTmem) {
    tc::tmem_alloc(&tmem_slot, kFusedTmemCols);
    tc::tc_fence_before();
  }
  // 1. scan (its first barrier publishes the TMEM base to its threads)
  if (threadIdx.x < scan::kThreads) scan::scan_cta<KDT, 1>(&tmap, &smap, F.scan, smem_raw, &tmem_slot);
  bool ok = grid_sync(F.bar, 1, F.scan.status, &s_ok);
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  tk::TkScratch& S = *reinterpret_cast<tk::TkScratch*>(sm);
  const int32_t rows = F.topk.rows;
  // 2. top-k collect
  if (ok && threadIdx.x < tk::kCollectThreads) {
    const int nv = F.collect_nseg * rows;
    for (int vb = blockIdx.x; vb < nv; vb += gridDim.x)
      tk::tk_collect_cta<2>(F.topk, F.collect_seg_len, vb % F.collect_nseg, vb / F.collect_nseg, S);
  }
  ok = ok && grid_sync(F.bar, 2, F.scan.status, &s_ok);
  // 3. top-k select, one row per CTA
  if (ok && threadIdx.x < kSelThreads) {
    uint32_t* fsm = reinterpret_cast<uint32_t*>(sm + kScratchBytes);
    for (int r = blockIdx.x; r < rows; r += gridDim.x) tk::tk_final_cta<kSelThreads, 3>(F.topk, r, fsm, S);
  }
  ok = ok && grid_sync(F.bar, 3, F.scan.status, &s_ok);
  // 4. attention
  if (ok) {
    const int ns = F.attn.nsplit;
    const int nv = ns * 2 * rows;
    for (int vb = blockIdx.x; vb < nv; vb += gridDim.x)
      attn::attn_cta(F.attn, smem_raw, vb % ns, (vb / ns) & 1, vb / (2 * ns), &tmem_slot);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == kWarpTmem) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_slot, kFusedTmemCols);
  }
}

template <int KDT>
size_t fused_smem(int64_t n_cols) {
  size_t b = scan::Cfg<KDT, 1>::kSmemBytes;
  if (static_cast<size_t>(attn::kSmemBytes) > b) b = attn::kSmemBytes;
  const size_t t = 1024 + kScratchBytes + tk::tk_final_smem(n_cols, kSelThreads);
  return t > b ? t : b;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

template <int KDT>
cudaError_t launch_t(const FusedParams& F, const CUtensorMap& tmap, const CUtensorMap& smap, cudaStream_t s) {
  const size_t smem = fused_smem<KDT>(F.topk.n_cols);
  auto kern = k_step_fused<KDT>;
  {
    cudaError_t e = ensure_dyn_smem(kern, smem);
    if (e != cudaSuccess) return e;
  }
  // every CTA must be resident at once (the grid barriers wait for all of them)
  int per_sm = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kFusedThreads, smem);
  if (e != cudaSuccess) return e;
  const int sms = num_sms();
  if (per_sm < 1 || sms < 1) return cudaErrorCooperativeLaunchTooLarge;
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(static_cast<unsigned>(sms));
  cfg.blockDim = dim3(kFusedThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tmap, smap, F);
}

// The attention's partials follow the top-k's zeroed head (histograms, list
// counters, control block); they overwrite bitmaps and candidates only after
// the select phase has finished with them.
size_t attn_part_bytes(int32_t rows, int32_t k, int ns, size_t* lse_bytes) {
  const size_t lse = tk::al256(static_cast<size_t>(rows) * ns * attn::kHeadsAll * sizeof(float));
  const size_t o = tk::al256(static_cast<size_t>(rows) * ns * attn::kHeadsAll * attn::kDv * sizeof(float));
  if (lse_bytes) *lse_bytes = lse;
  (void)k;
  return ns > 1 ? lse + o : 0;
}

}  // namespace

bool step_fused_supported(const ScoresArgs& sa, const AttnArgs& aa, int64_t n_cols) {
  return topk_v2_ok(n_cols) && scores_tc_fused_hist_ok(sa) && attn_tc_supported(aa) &&
         (sa.key_dtype == LSA_BF16 || sa.key_dtype == LSA_FP8_E4M3);
}

size_t step_fused_ws_bytes(int32_t rows, int64_t n_cols, int32_t k) {
  const size_t part = tk::tk_zero_bytes(rows) + attn_part_bytes(rows, k, attn::tc_nsplit(rows, k), nullptr);
  const size_t topk = tk::tk_ws_bytes(rows, n_cols);
  return part > topk ? part : topk;
}

cudaError_t launch_step_fused(const ScoresArgs& sa, const TopkArgs& ta, const AttnArgs& aa, cudaStream_t s) {
  const int32_t rows = ta.rows;
  if (rows == 0) return cudaSuccess;
  const tk::TkLayout L = tk::tk_layout(ta.ws, rows, ta.n_cols);
  FusedParams F;
  F.scan = sa;
  F.scan.hist12 = L.hist;
  F.topk = ta;
  F.topk.hist_ready = true;
  F.attn.a = aa;
  F.attn.nsplit = attn::tc_nsplit(rows, aa.k);
  const int chunks = (aa.k + attn::kChunk - 1) / attn::kChunk;
  F.attn.split_len = ((chunks + F.attn.nsplit - 1) / F.attn.nsplit) * attn::kChunk;
  size_t lse_bytes = 0;
  attn_part_bytes(rows, aa.k, F.attn.nsplit, &lse_bytes);
  uint8_t* part = static_cast<uint8_t*>(ta.ws) + tk::tk_zero_bytes(rows);
  F.attn.counters = reinterpret_cast<int*>(L.ctrl + tk::kCtrlInts);
  F.attn.part_lse = reinterpret_cast<float*>(part);
  F.attn.part_o = reinterpret_cast<float*>(part + lse_bytes);
  F.attn.merge = attn::kMergeInKernel;
  // the split CTAs of a row meet inside the attention phase: each must be a CTA of its own
  if (F.attn.nsplit > 1 && F.attn.nsplit * 2 * rows > num_sms()) return cudaErrorCooperativeLaunchTooLarge;
  const TopkPlan cp = topk_collect_plan(rows, ta.n_cols, num_sms());  // one segment per CTA
  F.collect_nseg = cp.nseg;
  F.collect_seg_len = cp.seg_len;
  F.bar = L.ctrl;
  CUtensorMap tmap, smap;
  cudaError_t e = scan_tc_maps(sa, &tmap, &smap);
  if (e != cudaSuccess) return e;
  // histograms, list counters, grid-barrier word and split counters start at zero
  e = cudaMemsetAsync(ta.ws, 0, tk::tk_zero_bytes(rows), s);
  if (e != cudaSuccess) return e;
  return sa.key_dtype == LSA_FP8_E4M3 ? launch_t<LSA_FP8_E4M3>(F, tmap, smap, s)
                                      : launch_t<LSA_BF16>(F, tmap, smap, s);
}

}  // namespace lsa
