// Exact top-k of fp32 score rows on an order-preserving 32-bit key.
//
// Keeps the k tokens with the largest scores in each row (MLI abstract, sentence 2):
//   * -0.0 compares equal to +0.0 (canonicalised before the key transform);
//   * -inf and NaN are never selected (they map to key 0, which is skipped);
//   * among equal scores the lower position is kept;
//   * the output holds min(k, #selectable) positions sorted ascending, then -1.
//
// Rows of up to 2^19 entries (every decode and prefill shape here) take three
// launches: a 12-bit histogram over segments of every row (all SMs), a collect
// pass that appends the positions above the threshold bin ("sure") and the
// (key, position) pairs inside it ("candidates") to per-row lists, and one CTA
// per row that finishes the radix select on the candidates in shared memory
// and writes the positions in order through a position bitmap.  If a
// threshold bin holds more candidates than the list keeps, that row's CTA
// re-reads its row instead.  Longer rows use five launches of segment-parallel
// radix passes (11 + 11 + 10 bits) with a count pass and an ordered compaction.
// Segments publish histograms and counts through global memory between
// launches, so no kernel waits on another CTA.
#include <math.h>

#include <map>
#include <mutex>
#include <tuple>

#include <string.h>

#include "common.cuh"
#include "host_util.h"
#include "internal.h"
#include "tc.cuh"
#include "topk_cluster.cuh"
#include "topk_sel.cuh"

namespace lsa {
namespace {

constexpr int kT = 256;            // threads per CTA
constexpr int kRound = kT * 4;     // elements per round (one float4 per thread)
constexpr int kBins1 = 2048, kBins2 = 2048, kBins3 = 1024;
constexpr int kHistStride = kBins1 + kBins2 + kBins3;


struct Row {
  int64_t n;       // valid entries of this row
  int64_t s0, s1;  // this CTA's segment [s0, s1)
};

__device__ __forceinline__ Row row_range(const TopkArgs& a, int r, int seg, int64_t seg_len) {
  int64_t n = a.n_cols;
  if (a.valid_len) {
    int64_t v = __ldg(a.valid_len + r);
    n = v < 0 ? 0 : (v < n ? v : n);
  }
  Row x;
  x.n = n;
  x.s0 = static_cast<int64_t>(seg) * seg_len;
  x.s1 = x.s0 + seg_len < n ? x.s0 + seg_len : n;
  return x;
}

// Loads the 4 keys of this thread for the round starting at `base` (positions
// >= n give key 0).  Rows start 16-byte aligned (ld % 4 == 0 is checked on the host).
__device__ __forceinline__ void load_keys(const float* row, int64_t base, int64_t n, uint32_t (&k)[4]) {
  const int64_t p = base + threadIdx.x * 4;
  if (p + 3 < n) {
    float4 v = __ldg(reinterpret_cast<const float4*>(row + p));
    k[0] = order_key(v.x); k[1] = order_key(v.y); k[2] = order_key(v.z); k[3] = order_key(v.w);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) k[j] = (p + j < n) ? order_key(__ldg(row + p + j)) : 0u;
  }
}

// Block-wide exclusive prefix sum of v (all threads), total in *total.
__device__ __forceinline__ int block_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kT / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kT / 32) warp_sums[lane] = w;  // inclusive
  }
  __syncthreads();
  const int before = warp ? warp_sums[warp - 1] : 0;
  *total = warp_sums[kT / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// Finds the bin holding the k_rem-th largest key of a histogram (bins ordered
// by key, so larger bins hold larger keys).  Returns bin (-1 if the histogram
// holds fewer than k_rem keys) and the rank inside it; *total = sum of bins.
struct Found {
  int bin;
  uint32_t rank;  // 1-based rank of the wanted key among the keys of `bin`
  uint32_t total;
};

template <int NB>
__device__ Found find_bin(const uint32_t* __restrict__ hist, uint32_t k_rem, int* sh) {
  constexpr int PER = NB / kT;  // bins per thread
  const int t = threadIdx.x;
  uint32_t v[PER];
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    v[i] = __ldcg(hist + t * PER + i);
    mine += v[i];
  }
  // suffix sums: keys held by threads t' > t (higher bins)
  int tot;
  int excl = block_excl_scan(static_cast<int>(mine), sh, &tot);
  uint32_t above = static_cast<uint32_t>(tot) - static_cast<uint32_t>(excl) - mine;
  __shared__ Found res;
  if (t == 0) res = Found{-1, 0u, static_cast<uint32_t>(tot)};
  __syncthreads();
  if (k_rem > 0 && above < k_rem && k_rem <= above + mine) {
    uint32_t cum = above;
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (cum + v[i] >= k_rem) {
        res.bin = t * PER + i;
        res.rank = k_rem - cum;
        break;
      }
      cum += v[i];
    }
  }
  __syncthreads();
  Found f = res;
  __syncthreads();
  return f;
}

struct Thresh {
  bool any;        // at least one key selected
  uint32_t keff;   // min(k, selectable)
  uint32_t T;      // key of the k-th selected element (valid for the last stage reached)
  uint32_t ties;   // how many keys equal to T are selected (final stage only)
  int b1, b2;
};

// Recomputes the threshold state from the histograms published so far.
template <int STAGES>
__device__ Thresh thresholds(const uint32_t* hist_row, int k, int* sh) {
  Thresh th{};
  Found f1 = find_bin<kBins1>(hist_row, 0xffffffffu, sh);  // only for the total
  uint32_t keff = f1.total < static_cast<uint32_t>(k) ? f1.total : static_cast<uint32_t>(k);
  th.keff = keff;
  th.any = keff > 0;
  if (!th.any) return th;
  f1 = find_bin<kBins1>(hist_row, keff, sh);
  th.b1 = f1.bin;
  if (STAGES == 1) return th;
  Found f2 = find_bin<kBins2>(hist_row + kBins1, f1.rank, sh);
  th.b2 = f2.bin;
  if (STAGES == 2) return th;
  Found f3 = find_bin<kBins3>(hist_row + kBins1 + kBins2, f2.rank, sh);
  th.T = (static_cast<uint32_t>(f1.bin) << 21) | (static_cast<uint32_t>(f2.bin) << 10) | static_cast<uint32_t>(f3.bin);
  th.ties = f3.rank;
  return th;
}

// PASS 1: histogram of bits [31:21]; PASS 2: bits [20:10] of keys in bin b1;
// PASS 3: bits [9:0] of keys with prefix (b1, b2).
template <int PASS>
__global__ void __launch_bounds__(kT) k_topk_hist(TopkArgs a, int64_t seg_len) {
  constexpr int NB = PASS == 3 ? kBins3 : kBins1;
  __shared__ uint32_t h[NB];
  __shared__ int sh[kT / 32];
  const int r = blockIdx.y, seg = blockIdx.x;
  const Row rr = row_range(a, r, seg, seg_len);
  if (rr.s0 >= rr.s1) return;
  uint32_t* hist_row = reinterpret_cast<uint32_t*>(a.ws) + static_cast<int64_t>(r) * kHistStride;
  uint32_t prefix = 0;
  if (PASS >= 2) {
    Thresh th = thresholds<PASS - 1>(hist_row, a.k, sh);
    if (!th.any) return;
    prefix = PASS == 2 ? static_cast<uint32_t>(th.b1) : ((static_cast<uint32_t>(th.b1) << 11) | th.b2);
  }
  for (int i = threadIdx.x; i < NB; i += kT) h[i] = 0;
  __syncthreads();
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  for (int64_t base = rr.s0; base < rr.s1; base += kRound) {
    uint32_t key[4];
    load_keys(row, base, rr.s1, key);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t x = key[j];
      if (x == 0u) continue;
      if (PASS == 1) atomicAdd(&h[x >> 21], 1u);
      else if (PASS == 2) { if ((x >> 21) == prefix) atomicAdd(&h[(x >> 10) & 2047u], 1u); }
      else { if ((x >> 10) == prefix) atomicAdd(&h[x & 1023u], 1u); }
    }
  }
  __syncthreads();
  uint32_t* dst = hist_row + (PASS == 1 ? 0 : PASS == 2 ? kBins1 : kBins1 + kBins2);
  for (int i = threadIdx.x; i < NB; i += kT)
    if (h[i]) atomicAdd(dst + i, h[i]);
}

__device__ __forceinline__ int32_t* seg_counts(const TopkArgs& a, int r, int nseg) {
  uint8_t* base = reinterpret_cast<uint8_t*>(a.ws) + static_cast<size_t>(a.rows) * kHistStride * 4;
  return reinterpret_cast<int32_t*>(base) + (static_cast<int64_t>(r) * nseg) * 2;
}

// PASS 4: per segment, the counts of keys > T and == T.
__global__ void __launch_bounds__(kT) k_topk_count(TopkArgs a, int64_t seg_len, int nseg) {
  __shared__ int sh[kT / 32];
  const int r = blockIdx.y, seg = blockIdx.x;
  const Row rr = row_range(a, r, seg, seg_len);
  if (rr.s0 >= rr.s1) return;
  const uint32_t* hist_row = reinterpret_cast<const uint32_t*>(a.ws) + static_cast<int64_t>(r) * kHistStride;
  Thresh th = thresholds<3>(hist_row, a.k, sh);
  if (!th.any) return;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  int gt = 0, eq = 0;
  for (int64_t base = rr.s0; base < rr.s1; base += kRound) {
    uint32_t key[4];
    load_keys(row, base, rr.s1, key);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      gt += key[j] > th.T;
      eq += key[j] == th.T;
    }
  }
  int tg, te;
  block_excl_scan(gt, sh, &tg);
  block_excl_scan(eq, sh, &te);
  if (threadIdx.x == 0) {
    int32_t* c = seg_counts(a, r, nseg) + seg * 2;
    c[0] = tg;
    c[1] = te;
  }
}

// PASS 5: ordered compaction of the selected positions, and -1 padding.
__global__ void __launch_bounds__(kT) k_topk_write(TopkArgs a, int64_t seg_len, int nseg) {
  __shared__ int sh[kT / 32];
  const int r = blockIdx.y, seg = blockIdx.x;
  const Row rr = row_range(a, r, seg, seg_len);
  int32_t* out = a.idx + static_cast<int64_t>(r) * a.k;
  if (rr.s0 >= rr.s1 && seg != 0) return;
  const uint32_t* hist_row = reinterpret_cast<const uint32_t*>(a.ws) + static_cast<int64_t>(r) * kHistStride;
  Thresh th = thresholds<3>(hist_row, a.k, sh);
  if (seg == 0)
    for (int i = static_cast<int>(th.keff) + threadIdx.x; i < a.k; i += kT) out[i] = -1;
  if (!th.any || rr.s0 >= rr.s1) return;
  // selected before this segment, and ties (== T) seen before it
  const int32_t* c = seg_counts(a, r, nseg);
  int sel_before = 0, eq_before = 0;
  for (int s = threadIdx.x; s < seg; s += kT) {
    sel_before += c[2 * s];
    eq_before += c[2 * s + 1];
  }
  // Ties (key == T) go to the lowest positions, so the earlier segments took
  // min(ties, keys == T before this segment) of them.
  int tsel, teq;
  block_excl_scan(sel_before, sh, &tsel);  // totals only
  block_excl_scan(eq_before, sh, &teq);
  const int ties = static_cast<int>(th.ties);
  int out_pos = tsel + (teq < ties ? teq : ties);  // positions already written by earlier segments
  int eq_seen = teq;                              // ties (== T) at lower positions
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  for (int64_t base = rr.s0; base < rr.s1; base += kRound) {
    uint32_t key[4];
    load_keys(row, base, rr.s1, key);
    int my_eq = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) my_eq += key[j] == th.T;
    int eq_tot;
    int eq_ex = block_excl_scan(my_eq, sh, &eq_tot);
    bool sel[4];
    int my_sel = 0, e = eq_seen + eq_ex;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      bool s = key[j] > th.T;
      if (key[j] == th.T) {
        s = e < ties;
        ++e;
      }
      sel[j] = s;
      my_sel += s;
    }
    int sel_tot;
    int sel_ex = block_excl_scan(my_sel, sh, &sel_tot);
    int o = out_pos + sel_ex;
    const int64_t p = base + threadIdx.x * 4;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (!sel[j]) continue;
      if (o < a.k) out[o] = static_cast<int32_t>(p + j);
      else record_error(a.status, LSA_ERR_BOUNDS, r, o);  // cannot happen if the counts agree
      ++o;
    }
    out_pos += sel_tot;
    eq_seen += eq_tot;
  }
}


// ============================================================ three-kernel path
using tk::kB1;
using tk::kCandCap;
using tk::TkLayout;
using tk::tk_layout;

// Histogram of key bits [31:20] per row (when the scan did not build it).
__global__ void __launch_bounds__(kT) k_tk_hist12(TopkArgs a, int64_t seg_len) {
  __shared__ uint32_t h[kB1];
  const int r = blockIdx.y, seg = blockIdx.x;
  const Row rr = row_range(a, r, seg, seg_len);
  if (rr.s0 >= rr.s1) return;
  for (int i = threadIdx.x; i < kB1; i += kT) h[i] = 0;
  __syncthreads();
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  for (int64_t base = rr.s0; base < rr.s1; base += kRound) {
    uint32_t key[4];
    load_keys(row, base, rr.s1, key);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (key[j]) atomicAdd(&h[key[j] >> 20], 1u);
  }
  __syncthreads();
  uint32_t* dst = tk_layout(a.ws, a.rows, a.n_cols).hist + static_cast<int64_t>(r) * kB1;
  for (int i = threadIdx.x; i < kB1; i += kT)
    if (h[i]) atomicAdd(dst + i, h[i]);
}

// Collect pass of segment blockIdx.x of row blockIdx.y; the row's last CTA to
// finish its segment then selects the row's k (a grid-wide order is not
// needed: each row waits only for its own segments, and no CTA waits at all).
__global__ void __launch_bounds__(tk::kCollectThreads, 2) k_tk_rows(TopkArgs a, int64_t seg_len, int nseg) {
  extern __shared__ __align__(16) uint32_t fsm[];
  __shared__ tk::TkScratch S;
  __shared__ int s_last;
  const int r = blockIdx.y;
  const tk::TkLayout L = tk::tk_layout(a.ws, a.rows, a.n_cols);
  if (a.wait_ctr) {
    // decode step, launched early: wait until every scan CTA has counted
    // itself (its scores and histogram counts written and fenced)
    if (threadIdx.x == 0) {
      s_last = 1;
      const uint64_t t0 = tc::globaltimer_ns();
      for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.wait_ctr) : "memory");
        if (v >= a.wait_target) break;
        if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) {
          record_error(a.status, LSA_ERR_TIMEOUT, r, 20);
          s_last = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __syncthreads();
    if (!s_last) return;
  } else {
    tc::griddep_wait();  // launched early in a decode step: the scores are complete from here on
  }
  tc::griddep_launch_dependents();
  if (threadIdx.x == 0) S.s_keff = 0;  // what an empty segment leaves (the row's last CTA may be one)
  __syncthreads();
  const bool collected = tk::tk_collect_cta<2>(a, seg_len, blockIdx.x, r, S, a.split_select);
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's bitmap words and candidates before its count
    const uint32_t done = atomicAdd(L.row_done + r, 1u);
    s_last = done == static_cast<uint32_t>(nseg - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();  // the other segments' writes, read through L2 by the select
  if (a.split_select) {
    // decode step: exact bitmap and segment offsets for the attention's own
    // compaction, or (when that cannot be done) the full select into idx
    // (its keff, threshold bin and rank are this CTA's own, from its collect)
    const bool split = collected && tk::tk_split_select<tk::kCollectThreads, 3>(
                                        a, r, nseg, seg_len, S.s_keff, static_cast<uint32_t>(S.s_bin), S.s_rank, fsm, S);
    if (!split) tk::tk_final_cta<tk::kCollectThreads, 3>(a, r, fsm, S);
    __threadfence();  // this thread's marks, offsets or selection writes
    __syncthreads();
    if (threadIdx.x == 0)
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(L.selready + r), "r"(split ? 1u : 2u) : "memory");
    return;
  }
  tk::tk_final_cta<tk::kCollectThreads, 3>(a, r, fsm, S);
  if (a.wait_ctr) {
    // decode step: the attention of row r may read its selection from now on
    __threadfence();  // this thread's selection writes
    __syncthreads();
    if (threadIdx.x == 0) asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(L.sel_done + r), "r"(1u) : "memory");
  }
}

// One row per thread-block cluster (rows up to tk::kClMaxCols positions): CTA
// blockIdx.x of the cluster collects segment blockIdx.x of row blockIdx.y and
// the cluster selects the row together (topk_cluster.cuh).  MAXSEG: the body
// for clusters of up to 8 CTAs, or of 9 to 16.
template <int MAXSEG>
__global__ void __launch_bounds__(tk::kClThreads, 2) k_tk_cluster(TopkArgs a, int64_t seg_len, int nseg) {
  extern __shared__ __align__(16) uint8_t csm[];
  __shared__ tk::TkScratch S;
  __shared__ int s_live;
  const int r = blockIdx.y;
  if (a.wait_ctr) {
    // decode step, launched early: wait until every scan CTA has counted
    // itself (its scores and histogram counts written and fenced)
    if (threadIdx.x == 0) {
      s_live = 1;
      const uint64_t t0 = tc::globaltimer_ns();
      for (;;) {
        uint32_t v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a.wait_ctr) : "memory");
        if (v >= a.wait_target) break;
        if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) {
          record_error(a.status, LSA_ERR_TIMEOUT, r, 20);
          s_live = 0;
          break;
        }
        __nanosleep(64);
      }
    }
  } else {
    tc::griddep_wait();  // launched early in a decode step: the scores are complete from here on
    if (threadIdx.x == 0) s_live = 1;
  }
  __syncthreads();
  tc::griddep_launch_dependents();
  // every CTA of the cluster reaches the cluster barriers, live or not
  tk::tk_cluster_row<2, MAXSEG>(a, r, static_cast<int>(tc::cluster_ctarank()), nseg, seg_len, csm, S, s_live != 0);
}

// The cluster kernel for clusters of nseg CTAs, its dynamic shared memory
// raised to `smem` and, above 8 CTAs, non-portable cluster sizes allowed.
using ClusterKernel = void (*)(TopkArgs, int64_t, int);
cudaError_t cluster_kernel(int nseg, size_t smem, ClusterKernel* out) {
  const bool big = tk::cl_maxseg(nseg) > tk::kClPortableSeg;
  ClusterKernel fn = big ? k_tk_cluster<tk::kClMaxSeg> : k_tk_cluster<tk::kClPortableSeg>;
  cudaError_t e = ensure_dyn_smem(fn, smem);
  if (e != cudaSuccess) return e;
  if (big) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  *out = fn;
  return cudaSuccess;
}

// Clusters of `nseg` k_tk_cluster CTAs (with `smem` bytes each) the current
// device keeps resident at once; queried once per (device, nseg, smem).
int cluster_capacity(int nseg, size_t smem) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  static std::mutex mu;
  static std::map<std::tuple<int, int, size_t>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(dev, nseg, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  ClusterKernel fn = nullptr;
  if (cluster_kernel(nseg, smem, &fn) == cudaSuccess) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(nseg), 1, 1);
    cfg.blockDim = dim3(tk::kClThreads);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = static_cast<unsigned>(nseg);
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) n = 0;
  }
  (void)cudaGetLastError();
  cache[key] = n;
  return n;
}

// The cluster plan of the one-cluster-per-row top-k for these sizes: the
// largest cluster (16, 8, 4, 2 CTAs, or 1) whose clusters for every row fit on
// the device at once (a cluster that waits for a second wave costs a whole row's
// time again).  nseg = 0: too many rows for one wave; the collect + select
// kernel takes them.
tk::ClPlan cluster_plan(int32_t rows, int64_t n_cols) {
  for (int cap = tk::kClMaxSeg; cap >= 1; cap /= 2) {
    const tk::ClPlan p = tk::cl_plan(n_cols, cap);
    if (p.nseg == 0) break;                 // fewer segments would exceed what a CTA stages
    if (p.nseg < cap && cap > 1) continue;  // the row is too short for this many segments
    if (static_cast<int64_t>(rows) <= cluster_capacity(p.nseg, tk::cl_smem(p.seg_len, p.nseg))) return p;
  }
  tk::ClPlan none;
  none.nseg = 0;
  none.seg_len = 0;
  return none;
}

// SMs of the current device (the plan's CTA target).
int device_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return kPlanSMs;
  }
  return n;
}

// Collect CTAs resident per SM with the select's shared memory (at most 2).
int rows_ctas_per_sm(size_t smem) {
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_tk_rows, tk::kCollectThreads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return 1;
  }
  return n < 1 ? 1 : (n > 2 ? 2 : n);
}

}  // namespace

TopkPlan topk_plan(int32_t rows, int64_t n_cols) {
  TopkPlan p;
  int64_t target = 4LL * kPlanSMs;
  int64_t want = rows > 0 ? (target + rows - 1) / rows : 1;
  int64_t max_seg = (n_cols + 4095) / 4096;
  if (max_seg < 1) max_seg = 1;
  int64_t nseg = want < max_seg ? want : max_seg;
  if (nseg < 1) nseg = 1;
  int64_t seg_len = (n_cols + nseg - 1) / nseg;
  seg_len = ((seg_len + kRound - 1) / kRound) * kRound;
  if (seg_len < kRound) seg_len = kRound;
  p.seg_len = seg_len;
  p.nseg = static_cast<int32_t>((n_cols + seg_len - 1) / seg_len);
  if (p.nseg < 1) p.nseg = 1;
  return p;
}

bool topk_v2_ok(int64_t n_cols) { return n_cols <= tk::kMaxBitmapCols; }

bool topk_cluster_ok(int64_t n_cols) { return n_cols <= tk::kClMaxCols; }

bool topk_cluster_planned(int32_t rows, int64_t n_cols) {
  return topk_v2_ok(n_cols) && topk_cluster_ok(n_cols) && cluster_plan(rows, n_cols).nseg > 0;
}

size_t topk_hist_zero_bytes(int32_t rows) { return tk::tk_zero_bytes(rows); }

// Shared memory of a k_tk_rows launch (raising the kernel's limit once) and
// its segment plan.
cudaError_t rows_plan(int32_t rows, int64_t n_cols, size_t* smem_out, TopkPlan* plan) {
  size_t smem = tk::tk_final_smem(n_cols, tk::kCollectThreads);
  if (tk::tk_split_smem() > smem) smem = tk::tk_split_smem();
  const cudaError_t e = ensure_dyn_smem(k_tk_rows, smem);
  if (e != cudaSuccess) return e;
  *smem_out = smem;
  *plan = topk_collect_plan(rows, n_cols, rows_ctas_per_sm(smem) * device_sms());
  return cudaSuccess;
}

bool topk_rows_plan(int32_t rows, int64_t n_cols, int* nseg, int64_t* seg_len) {
  size_t smem;
  TopkPlan p;
  if (rows_plan(rows, n_cols, &smem, &p) != cudaSuccess) {
    (void)cudaGetLastError();
    return false;
  }
  *nseg = p.nseg;
  *seg_len = p.seg_len;
  return true;
}

void topk_step_flags(void* ws, int32_t rows, int64_t n_cols, uint32_t** scan_done, uint32_t** sel_done,
                     int** scan_pool) {
  const tk::TkLayout L = tk::tk_layout(ws, rows, n_cols);
  *scan_done = L.scan_done;
  *sel_done = L.sel_done;
  if (scan_pool) *scan_pool = L.scan_pool;
}

size_t topk_ws_bytes(int32_t rows, int64_t n_cols, int32_t) {
  const size_t R = static_cast<size_t>(rows);
  if (topk_v2_ok(n_cols)) return tk::tk_ws_bytes(rows, n_cols);
  TopkPlan p = topk_plan(rows, n_cols);
  size_t b = R * kHistStride * 4 + R * p.nseg * 8;
  return (b + 255) / 256 * 256;
}

lsa_status topk_check_args(const float* scores, int64_t ld, int32_t rows, int64_t n_cols, int32_t k,
                           const int32_t* idx) {
  if (rows < 0 || k < 1 || n_cols < 0 || ld < n_cols || (ld % 4) != 0) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!scores || !idx || (reinterpret_cast<uintptr_t>(scores) & 15u) != 0)) return LSA_ERR_INVALID_ARG;
  if (rows > 65535) return LSA_ERR_UNSUPPORTED;
  if (n_cols > (1LL << 31) - 1) return LSA_ERR_UNSUPPORTED;
  return LSA_OK;
}

size_t topk_call_bytes(int32_t rows, int64_t n_cols, int32_t k) {
  return kStatusBytes + (topk_ws_bytes(rows, n_cols, k) + 255) / 256 * 256;
}

int topk_launches(int64_t n_cols) { return topk_v2_ok(n_cols) ? 2 : 5; }

// Segments of the collect pass: multiples of 8192 positions, about
// `target_ctas` CTAs in total (two per SM for the standalone launch, where two
// latency-bound CTAs share an SM; one per CTA of the fused step).
TopkPlan topk_collect_plan(int32_t rows, int64_t n_cols, int32_t target_ctas) {
  TopkPlan p;
  const int64_t rounds = (n_cols + tk::kColRound - 1) / tk::kColRound;
  int64_t want = (static_cast<int64_t>(target_ctas) + rows - 1) / (rows > 0 ? rows : 1);
  if (want > rounds) want = rounds;
  if (want < 1) want = 1;
  const int64_t per = (rounds + want - 1) / want;
  p.seg_len = per * tk::kColRound;
  p.nseg = static_cast<int32_t>((rounds + per - 1) / per);
  if (p.nseg < 1) p.nseg = 1;
  return p;
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  if (a.rows == 0 || a.k == 0) return cudaSuccess;
  TopkPlan p = topk_plan(a.rows, a.n_cols);
  dim3 grid(static_cast<unsigned>(p.nseg), static_cast<unsigned>(a.rows));
  if (topk_v2_ok(a.n_cols)) {
    cudaError_t e;
    if (!a.hist_ready) {
      e = cudaMemsetAsync(a.ws, 0, topk_hist_zero_bytes(a.rows), s);
      if (e != cudaSuccess) return e;
      k_tk_hist12<<<grid, kT, 0, s>>>(a, p.seg_len);
    }
    const tk::ClPlan clp = (topk_cluster_ok(a.n_cols) && !a.split_select && a.allow_cluster)
                               ? cluster_plan(a.rows, a.n_cols) : tk::ClPlan{0, 0};
    if (clp.nseg > 0) {
      const tk::ClPlan& cp = clp;
      // one cluster of up to 16 CTAs per row
      const size_t smem = tk::cl_smem(cp.seg_len, cp.nseg);
      ClusterKernel fn = nullptr;
      e = cluster_kernel(cp.nseg, smem, &fn);
      if (e != cudaSuccess) return e;
      cudaLaunchConfig_t cfg;
      memset(&cfg, 0, sizeof(cfg));
      cfg.gridDim = dim3(static_cast<unsigned>(cp.nseg), static_cast<unsigned>(a.rows));
      cfg.blockDim = dim3(tk::kClThreads);
      cfg.dynamicSmemBytes = smem;
      cfg.stream = s;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeClusterDimension;
      attr[0].val.clusterDim.x = static_cast<unsigned>(cp.nseg);
      attr[0].val.clusterDim.y = 1;
      attr[0].val.clusterDim.z = 1;
      attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[1].val.programmaticStreamSerializationAllowed = 1;
      cfg.attrs = attr;
      cfg.numAttrs = a.pdl ? 2 : 1;
      return cudaLaunchKernelEx(&cfg, fn, a, cp.seg_len, cp.nseg);
    }
    size_t smem;
    TopkPlan cp;
    e = rows_plan(a.rows, a.n_cols, &smem, &cp);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3(static_cast<unsigned>(cp.nseg), static_cast<unsigned>(a.rows));
    cfg.blockDim = dim3(tk::kCollectThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = a.pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_tk_rows, a, cp.seg_len, static_cast<int>(cp.nseg));
  }
  size_t hist_bytes = static_cast<size_t>(a.rows) * kHistStride * 4;
  cudaError_t e = cudaMemsetAsync(a.ws, 0, hist_bytes, s);
  if (e != cudaSuccess) return e;
  k_topk_hist<1><<<grid, kT, 0, s>>>(a, p.seg_len);
  k_topk_hist<2><<<grid, kT, 0, s>>>(a, p.seg_len);
  k_topk_hist<3><<<grid, kT, 0, s>>>(a, p.seg_len);
  k_topk_count<<<grid, kT, 0, s>>>(a, p.seg_len, p.nseg);
  k_topk_write<<<grid, kT, 0, s>>>(a, p.seg_len, p.nseg);
  return cudaGetLastError();
}

}  // namespace lsa

// ---------------------------------------------------------------------------
// Top-k without a caller workspace.
//
// Some callers cannot allocate device memory where they call the top-k: a
// plugin host whose enqueue path forbids allocation, a runtime whose device
// memory is entirely pre-reserved by another allocator, or a latency-critical
// loop that cannot afford cudaMalloc's implicit synchronisation.  For them the
// scratch of the five top-k passes lives in the fixed-size array below, which
// every GPU that loads this library holds until the process exits.

namespace lsa {
namespace {

constexpr size_t kStaticScratchBytes = 4u << 20;  // 4 MiB: status word + histograms, bitmaps, candidates

static __device__ __align__(256) uint8_t g_topk_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_topk_scratch on the current device (the host-side name of
// the array is only a stand-in and must never reach a kernel).  Looked up once
// per device, with that device current.
cudaError_t static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_ptr[dev] = p;
  }
  *out = g_scratch_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace lsa

extern "C" lsa_status lsa_topk_noalloc(const float* scores, int64_t ld, int32_t rows, const int32_t* valid_len,
                                       int64_t n_cols, int32_t k, int32_t* idx, lsa_stream_t stream) {
  using namespace lsa;
  const lsa_status st = topk_check_args(scores, ld, rows, n_cols, k, idx);
  if (st != LSA_OK) return st;
  if (topk_call_bytes(rows, n_cols, k) > kStaticScratchBytes) return LSA_ERR_UNSUPPORTED;  // beyond the static scratch
  if (rows == 0) return LSA_OK;
  void* base = nullptr;
  if (static_scratch(&base) != cudaSuccess) return LSA_ERR_CUDA;
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.rows = rows;
  a.valid_len = valid_len;
  a.n_cols = n_cols;
  a.k = k;
  a.idx = idx;
  a.ws = static_cast<uint8_t*>(base) + kStatusBytes;  // histograms are zeroed by launch_topk
  a.status = reinterpret_cast<DevStatus*>(base);
  a.hist_ready = false;
  return launch_topk(a, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess ? LSA_OK : LSA_ERR_CUDA;
}
