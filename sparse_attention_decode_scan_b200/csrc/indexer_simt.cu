// Lightning-indexer scores on CUDA cores (any H_I <= 64, d_I multiple of 8).
//
// I(s) = sum_h w[h] * ReLU(scale_s * q_idx[h] . K[s])   (DSA lightning indexer,
// DeepSeek-V3.2-Exp report; the pass over every cached token that precedes
// each layer, MLI abstract sentence 2).  One thread per cached position; the query
// row's H_I x d_I block and weights sit in shared memory as fp32.  This is the
// general-shape path (the tiny fp32 workload, odd head counts); the tensor-core
// kernel in indexer_tc.cu takes the 64 x 128 production shape.
#include <math.h>

#include "common.cuh"
#include "host_util.h"
#include "internal.h"

namespace lsa {
namespace {

constexpr int kThreads = 128;

template <int KDT, int QDT, int MAXH>
__global__ void __launch_bounds__(kThreads) k_scores_simt(ScoresArgs a) {
  extern __shared__ float smem[];
  const int H = a.H, dI = a.dI;
  float* q_s = smem;                 // [MAXH][dI]
  float* w_s = smem + MAXH * dI;     // [MAXH]
  const int r = blockIdx.y;
  const int t = threadIdx.x;
  const int64_t p = static_cast<int64_t>(blockIdx.x) * kThreads + t;

  int b = a.row_seq ? __ldg(a.row_seq + r) : r;
  int64_t vis = 0;
  bool row_ok = (b >= 0 && b < a.cache.batch);
  if (row_ok) {
    int64_t L = __ldg(a.cache.seq_lens + b);
    if (L < 0 || L > a.cache.max_len) {
      if (p == 0) record_error(a.status, LSA_ERR_BOUNDS, r, static_cast<int>(L));
      L = L < 0 ? 0 : a.cache.max_len;
    }
    vis = L;
    if (a.row_pos) {
      int64_t pp = static_cast<int64_t>(__ldg(a.row_pos + r)) + 1;
      vis = pp < vis ? (pp < 0 ? 0 : pp) : vis;
    }
  } else if (p == 0) {
    record_error(a.status, LSA_ERR_BOUNDS, r, b);
  }
  float* out = a.scores + static_cast<int64_t>(r) * a.ld;
  const int64_t tile0 = static_cast<int64_t>(blockIdx.x) * kThreads;
  if (tile0 >= vis) {  // block-uniform: nothing visible in this tile
    if (p < a.ld) out[p] = row_ok ? -INFINITY : NAN;
    return;
  }
  const int64_t qoff = static_cast<int64_t>(r) * H * dI;
  for (int i = t; i < MAXH * dI; i += kThreads)
    q_s[i] = (i < H * dI) ? load_elem<QDT>(a.q_idx, qoff + i) : 0.f;
  for (int h = t; h < MAXH; h += kThreads) w_s[h] = (h < H) ? __ldg(a.w + static_cast<int64_t>(r) * H + h) : 0.f;
  __syncthreads();
  if (p >= a.ld) return;
  if (p >= vis) {
    out[p] = -INFINITY;
    return;
  }
  CacheAddr ad{a.cache.block_table, a.cache.max_blocks, a.cache.block_size, a.cache.n_blocks, a.cache.max_len};
  const int64_t row = ad.row(b, p);
  if (row < 0) {
    record_error(a.status, LSA_ERR_BOUNDS, r, static_cast<int>(p));
    out[p] = NAN;
    return;
  }
  float acc[MAXH];
#pragma unroll
  for (int h = 0; h < MAXH; ++h) acc[h] = 0.f;
  const int64_t kbase = row * dI;
  for (int d = 0; d < dI; d += 8) {
    float kv[8];
    load8<KDT>(a.cache.idx_keys, kbase + d, kv);
#pragma unroll
    for (int h = 0; h < MAXH; ++h) {
      const float4* qq = reinterpret_cast<const float4*>(q_s + h * dI + d);
      const float4 x = qq[0], y = qq[1];
      float s = acc[h];
      s = fmaf(x.x, kv[0], s); s = fmaf(x.y, kv[1], s); s = fmaf(x.z, kv[2], s); s = fmaf(x.w, kv[3], s);
      s = fmaf(y.x, kv[4], s); s = fmaf(y.y, kv[5], s); s = fmaf(y.z, kv[6], s); s = fmaf(y.w, kv[7], s);
      acc[h] = s;
    }
  }
  const float sc = (KDT == LSA_FP8_E4M3) ? __ldg(a.cache.idx_key_scales + row) : 1.f;
  float score = 0.f;
#pragma unroll
  for (int h = 0; h < MAXH; ++h) score = fmaf(w_s[h], fmaxf(acc[h] * sc, 0.f), score);
  out[p] = score;
}

template <int KDT, int QDT, int MAXH>
cudaError_t launch_t(const ScoresArgs& a, cudaStream_t s) {
  size_t smem = (static_cast<size_t>(MAXH) * a.dI + MAXH) * sizeof(float);
  auto fn = k_scores_simt<KDT, QDT, MAXH>;
  if (smem > 48 * 1024) {
    cudaError_t e = ensure_dyn_smem(fn, smem);
    if (e != cudaSuccess) return e;
  }
  dim3 grid(static_cast<unsigned>((a.ld + kThreads - 1) / kThreads), static_cast<unsigned>(a.rows));
  fn<<<grid, kThreads, smem, s>>>(a);
  return cudaGetLastError();
}

template <int KDT, int QDT>
cudaError_t launch_h(const ScoresArgs& a, cudaStream_t s) {
  if (a.H <= 8) return launch_t<KDT, QDT, 8>(a, s);
  if (a.H <= 16) return launch_t<KDT, QDT, 16>(a, s);
  return launch_t<KDT, QDT, 64>(a, s);
}

template <int KDT>
cudaError_t launch_q(const ScoresArgs& a, cudaStream_t s) {
  if (a.q_dtype == LSA_F32) return launch_h<KDT, LSA_F32>(a, s);
  return launch_h<KDT, LSA_BF16>(a, s);
}

}  // namespace

cudaError_t launch_scores_simt(const ScoresArgs& a, cudaStream_t s) {
  if (a.rows == 0 || a.ld == 0) return cudaSuccess;
  switch (a.key_dtype) {
    case LSA_F32: return launch_q<LSA_F32>(a, s);
    case LSA_BF16: return launch_q<LSA_BF16>(a, s);
    default: return launch_q<LSA_FP8_E4M3>(a, s);
  }
}

}  // namespace lsa
