// Exact top-k of fp32 score rows on an order-preserving 32-bit key.
//
// Keeps the k highest-scoring tokens of each row (MLI abstract, sentence 2):
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

#include <mutex>

#include "common.cuh"
#include "internal.h"

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
constexpr int kB1 = kTopkBins1;     // 12-bit first digit
constexpr int kCandCap = 8192;     // candidates kept per row
constexpr int64_t kMaxBitmapCols = 1 << 19;
constexpr int kFinT = 1024;        // threads of the per-row CTA
constexpr int kWordElems = 32;     // positions per bitmap word (one thread's share of a round)
constexpr int kColRound = kT * kWordElems;  // positions per collect round (8192)

// Workspace: [rows][4096] first-digit histograms | [rows][words] bitmaps of the
// keys above the threshold bin | [rows] candidate counts | [rows][kCandCap]
// candidates (key, position).
struct TkLayout {
  uint32_t* hist;
  uint32_t* bitmap;
  uint32_t* ncand;
  uint2* cand;
  int64_t words;
};

__host__ __device__ inline size_t al256(size_t b) { return (b + 255) / 256 * 256; }

__host__ __device__ inline TkLayout tk_layout(void* ws, int32_t rows, int64_t n_cols) {
  TkLayout L;
  uint8_t* b = static_cast<uint8_t*>(ws);
  L.words = (n_cols + 31) / 32;
  L.hist = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * kB1 * 4);
  L.ncand = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * 4);
  L.bitmap = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * L.words * 4);
  L.cand = reinterpret_cast<uint2*>(b);
  return L;
}

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

// Threshold bin b1 of each row, then each thread takes 32 consecutive
// positions per round: the keys above b1 become one bitmap word (written once,
// no atomics) and the keys inside b1 are appended to the row's candidates
// (one atomic per CTA and round).  Segments are multiples of 8192 positions
// and cover [0, n_cols), so every bitmap word is written.
__global__ void __launch_bounds__(kT) k_tk_collect(TopkArgs a, int64_t seg_len) {
  __shared__ int sh[kT / 32];
  __shared__ uint32_t s_base;
  const int r = blockIdx.y, seg = blockIdx.x;
  int64_t n = a.n_cols;
  if (a.valid_len) {
    const int64_t v = __ldg(a.valid_len + r);
    n = v < 0 ? 0 : (v < n ? v : n);
  }
  const int64_t s0 = static_cast<int64_t>(seg) * seg_len;
  const int64_t s1 = s0 + seg_len < a.n_cols ? s0 + seg_len : a.n_cols;
  if (s0 >= s1) return;
  const TkLayout L = tk_layout(a.ws, a.rows, a.n_cols);
  const uint32_t* hist = L.hist + static_cast<int64_t>(r) * kB1;
  Found f = find_bin<kB1>(hist, 0xffffffffu, sh);
  const uint32_t keff = f.total < static_cast<uint32_t>(a.k) ? f.total : static_cast<uint32_t>(a.k);
  uint32_t b1 = 0xffffffffu;  // no selection: no bin qualifies
  if (keff > 0) {
    f = find_bin<kB1>(hist, keff, sh);
    b1 = static_cast<uint32_t>(f.bin);
  }
  uint32_t* bitmap = L.bitmap + static_cast<int64_t>(r) * L.words;
  uint2* cand = L.cand + static_cast<int64_t>(r) * kCandCap;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  for (int64_t base = s0; base < s1; base += kColRound) {
    const int64_t p0 = base + static_cast<int64_t>(threadIdx.x) * kWordElems;
    uint32_t key[kWordElems];
    if (p0 + kWordElems <= n) {
      const float4* src = reinterpret_cast<const float4*>(row + p0);
#pragma unroll
      for (int v = 0; v < kWordElems / 4; ++v) {
        const float4 x = __ldg(src + v);
        key[4 * v] = order_key(x.x); key[4 * v + 1] = order_key(x.y);
        key[4 * v + 2] = order_key(x.z); key[4 * v + 3] = order_key(x.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < kWordElems; ++e) key[e] = p0 + e < n ? order_key(__ldg(row + p0 + e)) : 0u;
    }
    uint32_t word = 0;
    int nc = 0;
#pragma unroll
    for (int e = 0; e < kWordElems; ++e) {
      const uint32_t bin = key[e] ? (key[e] >> 20) : 0xffffffffu;
      if (keff > 0 && key[e] && bin > b1) word |= 1u << e;
      nc += (keff > 0 && key[e] && bin == b1);
    }
    if (p0 < a.n_cols) bitmap[p0 / kWordElems] = word;
    int tot;
    const int off = block_excl_scan(nc, sh, &tot);
    if (threadIdx.x == 0) s_base = tot ? atomicAdd(L.ncand + r, static_cast<uint32_t>(tot)) : 0u;
    __syncthreads();
    uint32_t o = s_base + static_cast<uint32_t>(off);
    __syncthreads();
    if (nc) {
#pragma unroll
      for (int e = 0; e < kWordElems; ++e) {
        if (keff > 0 && key[e] && (key[e] >> 20) == b1) {
          if (o < static_cast<uint32_t>(kCandCap)) cand[o] = make_uint2(key[e], static_cast<uint32_t>(p0 + e));
          ++o;
        }
      }
    }
  }
}

// Block-wide (kFinT threads) exclusive scan.
__device__ __forceinline__ int fin_excl_scan(int v, int* warp_sums, int* total) {
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
    int w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const int before = warp ? warp_sums[warp - 1] : 0;
  *total = warp_sums[kFinT / 32 - 1];
  __syncthreads();
  return before + x - v;
}

// Bin of the rank-th largest key in a 1024-bin shared histogram (one bin per
// thread); returns the bin and the rank inside it through shared memory.
__device__ __forceinline__ void fin_find(const uint32_t* h, uint32_t rank, int* warp_sums, int* out_bin,
                                         uint32_t* out_rank) {
  const int t = threadIdx.x;
  const uint32_t v = h[t];
  int tot;
  const int excl = fin_excl_scan(static_cast<int>(v), warp_sums, &tot);
  const uint32_t above = static_cast<uint32_t>(tot - excl) - v;  // keys in higher bins
  if (v > 0 && above < rank && rank <= above + v) {
    *out_bin = t;
    *out_rank = rank - above;
  }
  __syncthreads();
}

// keeps the n lowest set bits of x
__device__ __forceinline__ uint32_t low_bits(uint32_t x, int n) {
  uint32_t y = 0;
  for (int i = 0; i < n && x; ++i) {
    const uint32_t b = x & (0u - x);
    y |= b;
    x ^= b;
  }
  return y;
}

// One CTA per row: keff and b1 from the histogram, the bitmap of the keys
// above b1 and the candidates in shared memory, a radix select on the
// candidates' low 20 bits (or, if they overflowed the list, on the row again),
// and an ordered compaction of the bitmap.
__global__ void __launch_bounds__(kFinT) k_tk_final(TopkArgs a) {
  extern __shared__ __align__(16) uint32_t fsm[];
  __shared__ int warp_sums[32];
  __shared__ int s_bin;
  __shared__ uint32_t s_rank;
  __shared__ uint32_t h[1024];
  const int r = blockIdx.x;
  const int t = threadIdx.x;
  const TkLayout L = tk_layout(a.ws, a.rows, a.n_cols);
  const int64_t nwords = L.words;
  uint32_t* bm = fsm;               // selected positions
  uint32_t* tb = fsm + nwords;      // positions equal to the threshold key
  uint2* cs = reinterpret_cast<uint2*>(fsm + 2 * nwords);  // candidates: 2*nwords words keep 8-byte alignment
  int32_t* out = a.idx + static_cast<int64_t>(r) * a.k;
  int64_t n = a.n_cols;
  if (a.valid_len) {
    const int64_t v = __ldg(a.valid_len + r);
    n = v < 0 ? 0 : (v < n ? v : n);
  }
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  // issue every independent load first
  const uint32_t* hist = L.hist + static_cast<int64_t>(r) * kB1;
  uint32_t hv[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) hv[i] = __ldcg(hist + t * 4 + i);
  const uint32_t n_cand = __ldcg(L.ncand + r);
  const uint32_t* gbm = L.bitmap + static_cast<int64_t>(r) * nwords;
  for (int64_t w = t; w < nwords; w += kFinT) {
    bm[w] = __ldcg(gbm + w);
    tb[w] = 0;
  }
  const bool overflow = n_cand > static_cast<uint32_t>(kCandCap);
  const int nc = overflow ? 0 : static_cast<int>(n_cand);
  for (int c = t; c < nc; c += kFinT) cs[c] = __ldcg(L.cand + static_cast<int64_t>(r) * kCandCap + c);
  // keff and the threshold bin (4 bins per thread)
  uint32_t keff, b1, rank1;
  {
    const uint32_t mine = hv[0] + hv[1] + hv[2] + hv[3];
    int total;
    const int excl = fin_excl_scan(static_cast<int>(mine), warp_sums, &total);
    keff = static_cast<uint32_t>(total) < static_cast<uint32_t>(a.k) ? static_cast<uint32_t>(total)
                                                                     : static_cast<uint32_t>(a.k);
    uint32_t cum = static_cast<uint32_t>(total - excl) - mine;
    if (keff > 0 && cum < keff && keff <= cum + mine) {
      for (int i = 3; i >= 0; --i) {
        if (cum + hv[i] >= keff) {
          s_bin = t * 4 + i;
          s_rank = keff - cum;
          break;
        }
        cum += hv[i];
      }
    }
    __syncthreads();
    b1 = static_cast<uint32_t>(s_bin);
    rank1 = s_rank;  // wanted rank inside bin b1
  }
  for (int i = static_cast<int>(keff) + t; i < a.k; i += kFinT) out[i] = -1;
  if (keff == 0) return;
  // radix select on bits [19:10] then [9:0] among the keys of bin b1
  uint32_t T = 0, ties = 0;
  for (int pass = 0; pass < 2; ++pass) {
    h[t] = 0;
    __syncthreads();
    const uint32_t shift = pass == 0 ? 10 : 0;
    const uint32_t pre_shift = pass == 0 ? 20 : 10;
    const uint32_t prefix = pass == 0 ? b1 : (T >> 10);
    if (!overflow) {
      for (int c = t; c < nc; c += kFinT) {
        const uint32_t key = cs[c].x;
        if ((key >> pre_shift) == prefix) atomicAdd(&h[(key >> shift) & 1023u], 1u);
      }
    } else {
      for (int64_t base = 0; base < n; base += kFinT * 4) {
        const int64_t p = base + t * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (p + j >= n) break;
          const uint32_t key = order_key(__ldg(row + p + j));
          if (key && (key >> pre_shift) == prefix) atomicAdd(&h[(key >> shift) & 1023u], 1u);
        }
      }
    }
    __syncthreads();
    if (t == 0) s_bin = -1;
    __syncthreads();
    fin_find(h, pass == 0 ? rank1 : ties, warp_sums, &s_bin, &s_rank);
    const uint32_t bb = static_cast<uint32_t>(s_bin);
    if (pass == 0) {
      T = (b1 << 20) | (bb << 10);
      ties = s_rank;
    } else {
      T |= bb;
      ties = s_rank;
    }
    __syncthreads();
  }
  // mark keys of bin b1 above T, and collect the keys equal to T
  if (!overflow) {
    for (int c = t; c < nc; c += kFinT) {
      const uint2 e = cs[c];
      if (e.x > T) atomicOr(&bm[e.y >> 5], 1u << (e.y & 31));
      else if (e.x == T) atomicOr(&tb[e.y >> 5], 1u << (e.y & 31));
    }
  } else {
    for (int64_t base = 0; base < n; base += kFinT * 4) {
      const int64_t p = base + t * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (p + j >= n) break;
        const uint32_t key = order_key(__ldg(row + p + j));
        if ((key >> 20) != b1) continue;
        const uint32_t q = static_cast<uint32_t>(p + j);
        if (key > T) atomicOr(&bm[q >> 5], 1u << (q & 31));
        else if (key == T) atomicOr(&tb[q >> 5], 1u << (q & 31));
      }
    }
  }
  __syncthreads();
  // ordered compaction: the lowest `ties` positions equal to T join the selection
  const int64_t per = (nwords + kFinT - 1) / kFinT;
  const int64_t w0 = t * per, w1 = (w0 + per < nwords) ? w0 + per : nwords;
  int my_ties = 0;
  for (int64_t w = w0; w < w1; ++w) my_ties += __popc(tb[w]);
  int tie_tot;
  int tie_before = fin_excl_scan(my_ties, warp_sums, &tie_tot);
  int my_sel = 0;
  for (int64_t w = w0; w < w1; ++w) {
    const uint32_t x = tb[w];
    const int px = __popc(x);
    const int take = static_cast<int>(ties) - tie_before;
    uint32_t add = 0;
    if (take > 0) add = take >= px ? x : low_bits(x, take);
    tie_before += px;
    const uint32_t merged = bm[w] | add;
    bm[w] = merged;
    my_sel += __popc(merged);
  }
  int sel_tot;
  int o = fin_excl_scan(my_sel, warp_sums, &sel_tot);
  for (int64_t w = w0; w < w1; ++w) {
    uint32_t x = bm[w];
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (o < a.k) out[o] = static_cast<int32_t>(w * 32 + b);
      else record_error(a.status, LSA_ERR_BOUNDS, r, o);  // cannot happen
      ++o;
    }
  }
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

bool topk_v2_ok(int64_t n_cols) { return n_cols <= kMaxBitmapCols; }

size_t topk_hist_zero_bytes(int32_t rows) {
  return al256(static_cast<size_t>(rows) * kB1 * 4) + al256(static_cast<size_t>(rows) * 4);
}

size_t topk_ws_bytes(int32_t rows, int64_t n_cols, int32_t) {
  const size_t R = static_cast<size_t>(rows);
  if (topk_v2_ok(n_cols))
    return topk_hist_zero_bytes(rows) + al256(R * ((n_cols + 31) / 32) * 4) + al256(R * kCandCap * 8);
  TopkPlan p = topk_plan(rows, n_cols);
  size_t b = R * kHistStride * 4 + R * p.nseg * 8;
  return (b + 255) / 256 * 256;
}

int topk_launches(int64_t n_cols) { return topk_v2_ok(n_cols) ? 3 : 5; }

// Segments of the collect pass: multiples of 8192 positions, about two CTAs
// per SM in total.
TopkPlan collect_plan(int32_t rows, int64_t n_cols) {
  TopkPlan p;
  const int64_t rounds = (n_cols + kColRound - 1) / kColRound;
  int64_t want = (2LL * kPlanSMs + rows - 1) / (rows > 0 ? rows : 1);
  if (want > rounds) want = rounds;
  if (want < 1) want = 1;
  const int64_t per = (rounds + want - 1) / want;
  p.seg_len = per * kColRound;
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
    const TopkPlan cp = collect_plan(a.rows, a.n_cols);
    k_tk_collect<<<dim3(static_cast<unsigned>(cp.nseg), static_cast<unsigned>(a.rows)), kT, 0, s>>>(a, cp.seg_len);
    const int64_t nwords = (a.n_cols + 31) / 32;
    const size_t smem = 2 * nwords * 4 + static_cast<size_t>(kCandCap) * 8;
    static size_t smem_set = 0;
    if (smem > 48 * 1024 && smem > smem_set) {
      e = cudaFuncSetAttribute(k_tk_final, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      smem_set = smem;
    }
    k_tk_final<<<a.rows, kFinT, smem, s>>>(a);
    return cudaGetLastError();
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
  if (rows < 0 || k < 1 || n_cols < 0 || ld < n_cols || (ld % 4) != 0) return LSA_ERR_INVALID_ARG;
  if (rows > 0 && (!scores || !idx || (reinterpret_cast<uintptr_t>(scores) & 15u) != 0)) return LSA_ERR_INVALID_ARG;
  if (n_cols > (1LL << 31) - 1) return LSA_ERR_UNSUPPORTED;
  const size_t need = kStatusBytes + topk_ws_bytes(rows, n_cols, k);
  if (need > kStaticScratchBytes) return LSA_ERR_UNSUPPORTED;  // beyond the static scratch
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
