// Sparse MQA over the selected KV rows on CUDA cores, split over the index
// list, with a log-sum-exp merge of the split partials.
//
// For every query row and head h: o[h] = sum_j softmax_j(scale * q[h] . KV[idx_j])
// * KV[idx_j][0:D_v] over the kept positions only (the layer attends only the
// k tokens the indexer kept, MLI abstract sentence 2; sparse attention reduces
// reads but not storage, LeanSparse episode page).  One warp per head, lanes
// over the row width; online softmax per split.  This is the general-shape path
// (the tiny fp32 workload); attn_tc.cu handles the 128-head x 576 production
// shape on tensor cores.  The merge kernel is shared by both paths.
#include <math.h>

#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kWarps = 8;   // heads per CTA
constexpr int kT = kWarps * 32;

struct SimtAttnParams {
  AttnArgs a;
  int nsplit;
  int split_len;
  float* part_o;    // [rows][nsplit][H][Dv]
  float* part_lse;  // [rows][nsplit][H]
};

template <int DT>
__device__ __forceinline__ void store_out(void* out, int64_t i, float v);
template <>
__device__ __forceinline__ void store_out<LSA_F32>(void* out, int64_t i, float v) {
  reinterpret_cast<float*>(out)[i] = v;
}
template <>
__device__ __forceinline__ void store_out<LSA_BF16>(void* out, int64_t i, float v) {
  reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16_rn(v);
}

template <int DT, int DPL>
__global__ void __launch_bounds__(kT) k_attn_simt(SimtAttnParams P) {
  const AttnArgs& a = P.a;
  const int split = blockIdx.x, hg = blockIdx.y, r = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = hg * kWarps + warp;
  if (h >= a.H) return;  // warp-uniform; no block barrier below
  const int b = a.row_seq ? __ldg(a.row_seq + r) : r;
  const bool row_ok = b >= 0 && b < a.cache.batch;
  int64_t L = row_ok ? __ldg(a.cache.seq_lens + b) : 0;
  if (row_ok && (L < 0 || L > a.cache.max_len)) L = L < 0 ? 0 : a.cache.max_len;
  if (!row_ok && lane == 0 && warp == 0 && split == 0) record_error(a.status, LSA_ERR_BOUNDS, r, b);

  float q[DPL], o[DPL];
  const int64_t qoff = (static_cast<int64_t>(r) * a.H + h) * a.D;
#pragma unroll
  for (int i = 0; i < DPL; ++i) {
    const int d = lane + 32 * i;
    q[i] = d < a.D ? load_elem<DT>(a.q, qoff + d) : 0.f;
    o[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  CacheAddr ad{a.cache.block_table, a.cache.max_blocks, a.cache.block_size, a.cache.n_blocks, a.cache.max_len};
  const int j0 = split * P.split_len;
  const int j1 = min(a.k, j0 + P.split_len);
  const int32_t* idx = a.idx + static_cast<int64_t>(r) * a.k;
  for (int j = j0; row_ok && j < j1; ++j) {
    const int32_t pos = __ldg(idx + j);
    if (pos < 0) continue;
    int64_t row = pos < L ? ad.row(b, pos) : -1;
    if (row < 0) {
      if (lane == 0 && h == 0) record_error(a.status, LSA_ERR_BOUNDS, r, pos);
      continue;
    }
    const int64_t base = row * a.D;
    float v[DPL];
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = lane + 32 * i;
      v[i] = d < a.D ? load_elem<DT>(a.cache.kv, base + d) : 0.f;
      s = fmaf(q[i], v[i], s);
    }
    s = warp_sum(s) * a.scale;
    const float mn = fmaxf(m, s);
    const float alpha = expf(m - mn);
    const float p = expf(s - mn);
    l = l * alpha + p;
#pragma unroll
    for (int i = 0; i < DPL; ++i) o[i] = o[i] * alpha + p * v[i];
    m = mn;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const float lse = l > 0.f ? m + logf(l) : -INFINITY;
  if (P.nsplit == 1) {
    const int64_t ooff = (static_cast<int64_t>(r) * a.H + h) * a.Dv;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = lane + 32 * i;
      if (d < a.Dv) store_out<DT>(a.out, ooff + d, o[i] * inv);
    }
    if (a.lse && lane == 0) a.lse[static_cast<int64_t>(r) * a.H + h] = lse;
  } else {
    const int64_t slot = (static_cast<int64_t>(r) * P.nsplit + split) * a.H + h;
#pragma unroll
    for (int i = 0; i < DPL; ++i) {
      const int d = lane + 32 * i;
      if (d < a.Dv) P.part_o[slot * a.Dv + d] = o[i] * inv;
    }
    if (lane == 0) P.part_lse[slot] = lse;
  }
}

// o = sum_s exp(lse_s - lse) * o_s, lse = log sum_s exp(lse_s): exact merge of
// softmax partials over disjoint parts of the index list.
template <int DT>
__global__ void __launch_bounds__(kT) k_lse_merge(AttnArgs a, int nsplit, const float* part_o,
                                                   const float* part_lse) {
  const int r = blockIdx.y;
  const int h = blockIdx.x * kWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (h >= a.H) return;
  float mx = -INFINITY;
  for (int s = 0; s < nsplit; ++s)
    mx = fmaxf(mx, part_lse[(static_cast<int64_t>(r) * nsplit + s) * a.H + h]);
  const int64_t ooff = (static_cast<int64_t>(r) * a.H + h) * a.Dv;
  if (mx == -INFINITY) {
    for (int d = lane; d < a.Dv; d += 32) store_out<DT>(a.out, ooff + d, 0.f);
    if (a.lse && lane == 0) a.lse[static_cast<int64_t>(r) * a.H + h] = -INFINITY;
    return;
  }
  float den = 0.f;
  for (int s = 0; s < nsplit; ++s)
    den += expf(part_lse[(static_cast<int64_t>(r) * nsplit + s) * a.H + h] - mx);
  const float inv = 1.f / den;
  for (int d = lane; d < a.Dv; d += 32) {
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s) {
      const int64_t slot = (static_cast<int64_t>(r) * nsplit + s) * a.H + h;
      const float wgt = expf(part_lse[slot] - mx);
      if (wgt > 0.f) acc = fmaf(wgt, part_o[slot * a.Dv + d], acc);
    }
    store_out<DT>(a.out, ooff + d, acc * inv);
  }
  if (a.lse && lane == 0) a.lse[static_cast<int64_t>(r) * a.H + h] = mx + logf(den);
}

int simt_nsplit(int32_t rows, int32_t H, int32_t k) {
  const int hg = (H + kWarps - 1) / kWarps;
  const int64_t ctas = static_cast<int64_t>(rows) * hg;
  int want = static_cast<int>((2LL * kPlanSMs + ctas - 1) / (ctas > 0 ? ctas : 1));
  int maxs = (k + 63) / 64;
  int n = want < maxs ? want : maxs;
  return n < 1 ? 1 : n;
}

template <int DT, int DPL>
cudaError_t launch_simt_t(const SimtAttnParams& P, cudaStream_t s) {
  dim3 grid(P.nsplit, (P.a.H + kWarps - 1) / kWarps, P.a.rows);
  k_attn_simt<DT, DPL><<<grid, kT, 0, s>>>(P);
  return cudaGetLastError();
}

template <int DT>
cudaError_t launch_simt_d(const SimtAttnParams& P, cudaStream_t s) {
  const int dpl = (P.a.D + 31) / 32;
  if (dpl <= 2) return launch_simt_t<DT, 2>(P, s);
  if (dpl <= 4) return launch_simt_t<DT, 4>(P, s);
  if (dpl <= 8) return launch_simt_t<DT, 8>(P, s);
  if (dpl <= 18) return launch_simt_t<DT, 18>(P, s);
  return launch_simt_t<DT, 32>(P, s);
}

}  // namespace

int attn_simt_launches(int32_t rows, int32_t H, int32_t k) { return simt_nsplit(rows, H, k) > 1 ? 2 : 1; }

size_t attn_simt_ws_bytes(int32_t rows, int32_t H, int32_t Dv, int32_t k) {
  const int ns = simt_nsplit(rows, H, k);
  if (ns == 1) return 0;
  size_t b = static_cast<size_t>(rows) * ns * H * (Dv + 1) * sizeof(float);
  return (b + 255) / 256 * 256;
}

cudaError_t launch_attn_simt(const AttnArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  SimtAttnParams P;
  P.a = a;
  P.nsplit = simt_nsplit(a.rows, a.H, a.k);
  P.split_len = (a.k + P.nsplit - 1) / P.nsplit;
  float* ws = reinterpret_cast<float*>(a.ws);
  P.part_o = ws;
  P.part_lse = ws + static_cast<size_t>(a.rows) * P.nsplit * a.H * a.Dv;
  cudaError_t e = a.dtype == LSA_F32 ? launch_simt_d<LSA_F32>(P, s) : launch_simt_d<LSA_BF16>(P, s);
  if (e != cudaSuccess || P.nsplit == 1) return e;
  return launch_lse_merge(a, P.nsplit, P.part_o, P.part_lse, s);
}

cudaError_t launch_lse_merge(const AttnArgs& a, int nsplit, const float* part_o, const float* part_lse,
                             cudaStream_t s) {
  dim3 grid((a.H + kWarps - 1) / kWarps, a.rows);
  if (a.dtype == LSA_F32)
    k_lse_merge<LSA_F32><<<grid, kT, 0, s>>>(a, nsplit, part_o, part_lse);
  else
    k_lse_merge<LSA_BF16><<<grid, kT, 0, s>>>(a, nsplit, part_o, part_lse);
  return cudaGetLastError();
}

}  // namespace lsa
