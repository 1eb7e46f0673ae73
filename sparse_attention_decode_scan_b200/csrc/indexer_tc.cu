// Lightning-indexer scan on the sm_100a tensor cores: the standalone kernel
// (one persistent CTA per SM around the CTA body of scan_tc.cuh) and its host
// side (tensor maps, launch, support checks).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <string.h>

#include "common.cuh"
#include "host_util.h"
#include "internal.h"
#include "tc.cuh"

#include "scan_tc.cuh"

namespace lsa {
namespace {

using namespace scan;

template <int KDT, int QB, bool GATHER = false, int EG = 1>
__global__ void __launch_bounds__(scan_threads<EG>(), 1) k_scan_tc(const __grid_constant__ CUtensorMap tmap,
                                                                   const __grid_constant__ CUtensorMap smap,
                                                                   const ScoresArgs a) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint32_t tmem_slot;
  if ((threadIdx.x >> 5) == kWarpMma) {
    tc::tmem_alloc(&tmem_slot, Cfg<KDT, QB, GATHER>::kTmemCols);
    tc::tc_fence_before();
  }
  scan_cta<KDT, QB, GATHER, EG>(&tmap, &smap, a, smem_raw, &tmem_slot);
  if ((threadIdx.x >> 5) == kWarpMma) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_slot, Cfg<KDT, QB, GATHER>::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return kPlanSMs;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return kPlanSMs;
  return n;
}

int64_t key_rows(const ScoresArgs& a) {
  return a.cache.block_size > 0 ? a.cache.n_blocks * a.cache.block_size
                                : static_cast<int64_t>(a.cache.batch) * a.cache.max_len;
}

// Tensor maps of the scan: the key rows as 4-byte elements in 64-row boxes of
// one 128-byte K block, and (FP8) the key scales as a 1-D tensor.
cudaError_t make_maps(const ScoresArgs& a, CUtensorMap* tmap_out, CUtensorMap* smap_out) {
  auto fn = encode_fn();
  if (!fn) return cudaErrorNotSupported;
  CUtensorMap& tmap = *tmap_out;
  CUtensorMap& smap = *smap_out;
  const bool fp8 = a.key_dtype == LSA_FP8_E4M3;
  // The key rows are moved as opaque 4-byte elements (the 128-byte swizzle
  // works on bytes, so the shared-memory image is the same for bf16 and e4m3);
  // wider elements make fewer TMA element steps per byte.
  const int row_bytes = kDim * (fp8 ? 1 : 2);
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(row_bytes / 4), static_cast<cuuint64_t>(key_rows(a))};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(row_bytes)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kBoxX), static_cast<cuuint32_t>(kBoxRows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(&tmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2,
                  const_cast<void*>(a.cache.idx_keys), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  memset(&smap, 0, sizeof(smap));
  if (fp8) {  // FP8 key scales as a 1-D tensor over the same flat key rows
    const cuuint64_t sdims[1] = {static_cast<cuuint64_t>(key_rows(a))};
    const cuuint64_t sstrides[1] = {4};  // unused for rank 1
    const cuuint32_t sbox[1] = {static_cast<cuuint32_t>(kScaleBox)};
    const cuuint32_t sestr[1] = {1};
    r = fn(&smap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 1, const_cast<float*>(a.cache.idx_key_scales), sdims, sstrides,
           sbox, sestr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return cudaErrorInvalidValue;
  }
  return cudaSuccess;
}

// Epilogue groups: two groups of epilogue warps take alternate tiles.  The
// per-tile epilogue (TMEM loads, the ReLU-weighted head sums, the score
// stores and histogram counts) is the longest stage of the SM-side pipeline:
// with the key loads taken out, the bf16 decode scan still needed 132 of its
// 142 us with one group.  Two groups shorten the B=32 decode step by about
// 2.5 us (the scan's CTAs end closer together).
template <int KDT, int QB>
constexpr int epi_groups() { return 2; }

template <int KDT, int QB>
cudaError_t launch_t(const ScoresArgs& a, cudaStream_t s) {
  using C = Cfg<KDT, QB>;
  constexpr int EG = epi_groups<KDT, QB>();
  CUtensorMap tmap, smap;
  cudaError_t me = make_maps(a, &tmap, &smap);
  if (me != cudaSuccess) return me;
  auto kern = k_scan_tc<KDT, QB, false, EG>;
  cudaError_t e = ensure_dyn_smem(kern, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.grid > 0 ? a.grid : num_sms());
  if (a.pdl) {
    // a programmatic dependent: its CTAs take SMs as the kernel before frees them
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(scan_threads<EG>());
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr.val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, tmap, smap, a);
  }
  kern<<<grid, scan_threads<EG>(), C::kSmemBytes, s>>>(tmap, smap, a);
  return cudaGetLastError();
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

bool scores_tc_shape_ok(int32_t key_dtype, int32_t q_dtype, int32_t H, int32_t dI, int32_t block_size) {
  return (key_dtype == LSA_BF16 || key_dtype == LSA_FP8_E4M3) && q_dtype == LSA_BF16 && H == kHeads &&
         dI == kDim && (block_size == 0 || block_size % kBoxRows == 0);
}

int scores_tc_launches(bool) { return 1; }

bool scores_tc_supported(const ScoresArgs& a) {
  if (!scores_tc_shape_ok(a.key_dtype, a.q_dtype, a.H, a.dI, a.cache.block_size)) return false;
  if (!aligned16(a.cache.idx_keys) || !aligned16(a.q_idx) || !aligned16(a.w)) return false;
  const int64_t kr = key_rows(a);
  if (kr <= 0 || kr >= (1LL << 31)) return false;
  if (a.cache.max_len >= (1LL << 31)) return false;  // positions are kept as 32-bit integers
  if (a.key_dtype == LSA_FP8_E4M3 && (!a.cache.idx_key_scales || !aligned16(a.cache.idx_key_scales))) return false;
  return true;
}

size_t scores_tc_ws_bytes(int32_t, bool) { return 0; }

bool scores_tc_fused_hist_ok(const ScoresArgs& a) { return a.row_pos == nullptr && scores_tc_supported(a); }

bool scores_tc_pool_ok(const ScoresArgs& a) {
  // tile indices and row starts are kept as 32-bit integers
  const int64_t tiles_max = static_cast<int64_t>(a.rows) * ((a.cache.max_len + kTile - 1) / kTile);
  return a.row_pos == nullptr && a.cand == nullptr && a.rows <= kPoolRows && tiles_max < (1LL << 31) &&
         scores_tc_supported(a);
}

cudaError_t scan_tc_maps(const ScoresArgs& a, CUtensorMap* tmap, CUtensorMap* smap) { return make_maps(a, tmap, smap); }

int scan_tc_grid() { return num_sms(); }

bool candidate_scores_tc_supported(const ScoresArgs& a) {
  if (!a.cand || a.cand_ld < 0) return false;
  if (a.key_dtype != LSA_BF16 || a.q_dtype != LSA_BF16 || a.H != kHeads || a.dI != kDim) return false;
  if (!aligned16(a.cache.idx_keys) || !aligned16(a.q_idx) || !aligned16(a.w)) return false;
  const int64_t kr = key_rows(a);
  return kr > 0 && kr < (1LL << 31);
}

// Candidate re-scoring: the scan's CTA body with the gathering producer (no
// tensor maps: the rows are copied by cp.async).
cudaError_t launch_candidate_scores_tc(const ScoresArgs& a, cudaStream_t s) {
  using C = Cfg<LSA_BF16, 1, true>;
  auto kern = k_scan_tc<LSA_BF16, 1, true, 1>;
  cudaError_t e = ensure_dyn_smem(kern, C::kSmemBytes);
  if (e != cudaSuccess) return e;
  CUtensorMap none;
  memset(&none, 0, sizeof(none));
  kern<<<num_sms(), kThreads, C::kSmemBytes, s>>>(none, none, a);
  return cudaGetLastError();
}

cudaError_t launch_scores_tc(const ScoresArgs& a, cudaStream_t s) {
  const bool causal = a.row_pos != nullptr;
  if (a.key_dtype == LSA_FP8_E4M3) return causal ? launch_t<LSA_FP8_E4M3, 2>(a, s) : launch_t<LSA_FP8_E4M3, 1>(a, s);
  return causal ? launch_t<LSA_BF16, 4>(a, s) : launch_t<LSA_BF16, 1>(a, s);
}

}  // namespace lsa
