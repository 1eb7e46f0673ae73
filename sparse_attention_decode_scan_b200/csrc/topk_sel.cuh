// Top-k of rows of up to 2^19 scores: the device code of the collect pass and
// of the per-row select, shared by the standalone top-k kernels and the fused
// decode step.  Both are CTA bodies generic in their thread count NT and use a
// named barrier, so a block may hold more threads than take part.
//
// Exact top-k on an order-preserving 32-bit key (MLI abstract, sentence 2:
// the k best-scored tokens are kept): -0.0 equals +0.0, -inf and NaN are
// never selected, among equal scores the lower position wins, and a row's
// output is its min(k, #selectable) positions in ascending order, then -1.
#pragma once

#include "common.cuh"
#include "internal.h"

namespace lsa {
namespace tk {

constexpr int kB1 = kTopkBins1;          // 12-bit first digit (key bits [31:20])
constexpr int kCandCap = 8192;           // candidates kept per row
constexpr int64_t kMaxBitmapCols = 1 << 19;
constexpr int kWordElems = 32;           // positions per bitmap word (one thread's share of a round)
constexpr int kCollectThreads = 256;
constexpr int kColRound = kCollectThreads * kWordElems;  // positions per collect round (8192)
constexpr int kCtrlInts = 64;            // control words of the fused step (grid barrier) before the counters

__host__ __device__ inline size_t al256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace: [rows][4096] first-digit histograms | [rows] candidate counts |
// control block (fused step: grid-barrier word, attention split counters) |
// [rows][words] bitmaps of the keys above the threshold bin | [rows][kCandCap]
// candidates (key, position).  The first three are zeroed before each use.
struct TkLayout {
  uint32_t* hist;
  uint32_t* ncand;
  uint32_t* ctrl;
  uint32_t* bitmap;
  uint2* cand;
  int64_t words;
};

__host__ __device__ inline size_t tk_ctrl_bytes(int32_t rows) {
  return al256((static_cast<size_t>(kCtrlInts) + 2 * static_cast<size_t>(rows)) * 4);
}

__host__ __device__ inline size_t tk_zero_bytes(int32_t rows) {
  return al256(static_cast<size_t>(rows) * kB1 * 4) + al256(static_cast<size_t>(rows) * 4) + tk_ctrl_bytes(rows);
}

__host__ __device__ inline TkLayout tk_layout(void* ws, int32_t rows, int64_t n_cols) {
  TkLayout L;
  uint8_t* b = static_cast<uint8_t*>(ws);
  L.words = (n_cols + 31) / 32;
  L.hist = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * kB1 * 4);
  L.ncand = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * 4);
  L.ctrl = reinterpret_cast<uint32_t*>(b);
  b += tk_ctrl_bytes(rows);
  L.bitmap = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * L.words * 4);
  L.cand = reinterpret_cast<uint2*>(b);
  return L;
}

__host__ __device__ inline size_t tk_ws_bytes(int32_t rows, int64_t n_cols) {
  const size_t R = static_cast<size_t>(rows);
  return tk_zero_bytes(rows) + al256(R * ((n_cols + 31) / 32) * 4) + al256(R * kCandCap * 8);
}

// Shared scratch of the bodies (static in the standalone kernels, carved from
// dynamic shared memory in the fused step).
struct TkScratch {
  int warp_sums[32];
  int s_bin;
  uint32_t s_rank;
  uint32_t s_base;
  uint32_t h[1024];
};

template <int NT, int ID>
__device__ __forceinline__ void tk_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(ID), "n"(NT) : "memory");
}

// Exclusive prefix sum over the NT threads, total in *total.
template <int NT, int ID>
__device__ __forceinline__ int tk_excl_scan(int v, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  tk_sync<NT, ID>();
  if (warp == 0) {
    int w = lane < NT / 32 ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < NT / 32) warp_sums[lane] = w;  // inclusive
  }
  tk_sync<NT, ID>();
  const int before = warp ? warp_sums[warp - 1] : 0;
  *total = warp_sums[NT / 32 - 1];
  tk_sync<NT, ID>();
  return before + x - v;
}

// Bin (of NB, each thread holding NB/NT consecutive bins v[]) that holds the
// rank-th largest key, and the rank inside it, written to S.s_bin / S.s_rank
// by the thread that finds it.  Returns the histogram's total.
template <int NT, int ID, int NB>
__device__ __forceinline__ uint32_t tk_find(const uint32_t (&v)[NB / NT], uint32_t rank, TkScratch& S,
                                            bool use_total_as_rank) {
  constexpr int PER = NB / NT;
  uint32_t mine = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) mine += v[i];
  int tot;
  const int excl = tk_excl_scan<NT, ID>(static_cast<int>(mine), S.warp_sums, &tot);
  if (use_total_as_rank) rank = static_cast<uint32_t>(tot) < rank ? static_cast<uint32_t>(tot) : rank;
  uint32_t cum = static_cast<uint32_t>(tot - excl) - mine;  // keys in higher bins than this thread's
  if (rank > 0 && cum < rank && rank <= cum + mine) {
#pragma unroll
    for (int i = PER - 1; i >= 0; --i) {
      if (cum + v[i] >= rank) {
        S.s_bin = static_cast<int>(threadIdx.x) * PER + i;
        S.s_rank = rank - cum;
        break;
      }
      cum += v[i];
    }
  }
  tk_sync<NT, ID>();
  return static_cast<uint32_t>(tot);
}

// The collect pass for segment `seg` of row r: threshold bin b1 of the row from
// its first-digit histogram, then each thread takes 32 consecutive positions
// per round: the keys above b1 become one bitmap word (written once, no
// atomics) and the keys inside b1 are appended to the row's candidates (one
// atomic per CTA and round).  Segments are multiples of kColRound positions and
// cover [0, n_cols), so every bitmap word is written.
template <int ID>
__device__ void tk_collect_cta(const TopkArgs& a, int64_t seg_len, int seg, int r, TkScratch& S) {
  constexpr int NT = kCollectThreads;
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
  uint32_t hv[kB1 / NT];
#pragma unroll
  for (int i = 0; i < kB1 / NT; ++i) hv[i] = __ldcg(hist + threadIdx.x * (kB1 / NT) + i);
  const uint32_t total = tk_find<NT, ID, kB1>(hv, static_cast<uint32_t>(a.k), S, true);
  const uint32_t keff = total < static_cast<uint32_t>(a.k) ? total : static_cast<uint32_t>(a.k);
  const uint32_t b1 = keff > 0 ? static_cast<uint32_t>(S.s_bin) : 0xffffffffu;  // none: no bin qualifies
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
        const float4 x = __ldcg(src + v);  // coherent: the fused step writes the scores in the same launch
        key[4 * v] = order_key(x.x); key[4 * v + 1] = order_key(x.y);
        key[4 * v + 2] = order_key(x.z); key[4 * v + 3] = order_key(x.w);
      }
    } else {
#pragma unroll
      for (int e = 0; e < kWordElems; ++e) key[e] = p0 + e < n ? order_key(__ldcg(row + p0 + e)) : 0u;
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
    const int off = tk_excl_scan<NT, ID>(nc, S.warp_sums, &tot);
    if (threadIdx.x == 0) S.s_base = tot ? atomicAdd(L.ncand + r, static_cast<uint32_t>(tot)) : 0u;
    tk_sync<NT, ID>();
    uint32_t o = S.s_base + static_cast<uint32_t>(off);
    tk_sync<NT, ID>();
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

// Shared memory of the select body besides TkScratch: two bitmaps and the candidates.
__host__ __device__ inline size_t tk_final_smem(int64_t n_cols) {
  return 2 * static_cast<size_t>((n_cols + 31) / 32) * 4 + static_cast<size_t>(kCandCap) * 8;
}

// The select of row r: keff and b1 from the histogram, the bitmap of the keys
// above b1 and the candidates in shared memory (fsm, tk_final_smem bytes, 16-byte
// aligned), a radix select on the candidates' low 20 bits (or, if they
// overflowed the list, on the row again), and an ordered compaction of the bitmap.
template <int NT, int ID>
__device__ void tk_final_cta(const TopkArgs& a, int r, uint32_t* fsm, TkScratch& S) {
  const int t = threadIdx.x;
  const TkLayout L = tk_layout(a.ws, a.rows, a.n_cols);
  const int64_t nwords = L.words;
  uint32_t* bm = fsm;               // selected positions
  uint32_t* tb = fsm + nwords;      // positions equal to the threshold key
  uint2* cs = reinterpret_cast<uint2*>(fsm + 2 * nwords);  // 2*nwords words keep 8-byte alignment
  int32_t* out = a.idx + static_cast<int64_t>(r) * a.k;
  int64_t n = a.n_cols;
  if (a.valid_len) {
    const int64_t v = __ldg(a.valid_len + r);
    n = v < 0 ? 0 : (v < n ? v : n);
  }
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  // issue every independent load first
  const uint32_t* hist = L.hist + static_cast<int64_t>(r) * kB1;
  constexpr int HB = kB1 / NT;
  uint32_t hv[HB];
#pragma unroll
  for (int i = 0; i < HB; ++i) hv[i] = __ldcg(hist + t * HB + i);
  const uint32_t n_cand = __ldcg(L.ncand + r);
  const uint32_t* gbm = L.bitmap + static_cast<int64_t>(r) * nwords;
  for (int64_t w = t; w < nwords; w += NT) {
    bm[w] = __ldcg(gbm + w);
    tb[w] = 0;
  }
  const bool overflow = n_cand > static_cast<uint32_t>(kCandCap);
  const int nc = overflow ? 0 : static_cast<int>(n_cand);
  for (int c = t; c < nc; c += NT) cs[c] = __ldcg(L.cand + static_cast<int64_t>(r) * kCandCap + c);
  // keff and the threshold bin
  const uint32_t total = tk_find<NT, ID, kB1>(hv, static_cast<uint32_t>(a.k), S, true);
  const uint32_t keff = total < static_cast<uint32_t>(a.k) ? total : static_cast<uint32_t>(a.k);
  const uint32_t b1 = static_cast<uint32_t>(S.s_bin);
  const uint32_t rank1 = S.s_rank;  // wanted rank inside bin b1
  for (int i = static_cast<int>(keff) + t; i < a.k; i += NT) out[i] = -1;
  if (keff == 0) return;
  // radix select on bits [19:10] then [9:0] among the keys of bin b1
  uint32_t T = 0, ties = 0;
  for (int pass = 0; pass < 2; ++pass) {
    for (int i = t; i < 1024; i += NT) S.h[i] = 0;
    tk_sync<NT, ID>();
    const uint32_t shift = pass == 0 ? 10 : 0;
    const uint32_t pre_shift = pass == 0 ? 20 : 10;
    const uint32_t prefix = pass == 0 ? b1 : (T >> 10);
    if (!overflow) {
      for (int c = t; c < nc; c += NT) {
        const uint32_t key = cs[c].x;
        if ((key >> pre_shift) == prefix) atomicAdd(&S.h[(key >> shift) & 1023u], 1u);
      }
    } else {
      for (int64_t base = 0; base < n; base += NT * 4) {
        const int64_t p = base + t * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if (p + j >= n) break;
          const uint32_t key = order_key(__ldcg(row + p + j));
          if (key && (key >> pre_shift) == prefix) atomicAdd(&S.h[(key >> shift) & 1023u], 1u);
        }
      }
    }
    tk_sync<NT, ID>();
    uint32_t hl[1024 / NT];
#pragma unroll
    for (int i = 0; i < 1024 / NT; ++i) hl[i] = S.h[t * (1024 / NT) + i];
    tk_find<NT, ID, 1024>(hl, pass == 0 ? rank1 : ties, S, false);
    const uint32_t bb = static_cast<uint32_t>(S.s_bin);
    if (pass == 0) {
      T = (b1 << 20) | (bb << 10);
      ties = S.s_rank;
    } else {
      T |= bb;
      ties = S.s_rank;
    }
    tk_sync<NT, ID>();
  }
  // mark keys of bin b1 above T, and collect the keys equal to T
  if (!overflow) {
    for (int c = t; c < nc; c += NT) {
      const uint2 e = cs[c];
      if (e.x > T) atomicOr(&bm[e.y >> 5], 1u << (e.y & 31));
      else if (e.x == T) atomicOr(&tb[e.y >> 5], 1u << (e.y & 31));
    }
  } else {
    for (int64_t base = 0; base < n; base += NT * 4) {
      const int64_t p = base + t * 4;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (p + j >= n) break;
        const uint32_t key = order_key(__ldcg(row + p + j));
        if ((key >> 20) != b1) continue;
        const uint32_t q = static_cast<uint32_t>(p + j);
        if (key > T) atomicOr(&bm[q >> 5], 1u << (q & 31));
        else if (key == T) atomicOr(&tb[q >> 5], 1u << (q & 31));
      }
    }
  }
  tk_sync<NT, ID>();
  // ordered compaction: the lowest `ties` positions equal to T join the selection
  const int64_t per = (nwords + NT - 1) / NT;
  const int64_t w0 = t * per, w1 = (w0 + per < nwords) ? w0 + per : nwords;
  int my_ties = 0;
  for (int64_t w = w0; w < w1; ++w) my_ties += __popc(tb[w]);
  int tie_tot;
  int tie_before = tk_excl_scan<NT, ID>(my_ties, S.warp_sums, &tie_tot);
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
  int o = tk_excl_scan<NT, ID>(my_sel, S.warp_sums, &sel_tot);
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
  tk_sync<NT, ID>();  // shared memory free for the caller's next use
}

}  // namespace tk
}  // namespace lsa
