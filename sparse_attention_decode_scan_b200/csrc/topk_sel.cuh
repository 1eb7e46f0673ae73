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
constexpr int kMaxSeg = static_cast<int>(kMaxBitmapCols / kColRound);  // collect segments per row at most
constexpr int kTieCap = 256;             // keys equal to the threshold a split select ranks itself

__host__ __device__ inline size_t al256(size_t b) { return (b + 255) / 256 * 256; }

// Workspace: [rows][4096] first-digit histograms | [rows] candidate counts |
// control block (fused step: grid-barrier word; scan CTAs finished; attention
// split counters; per-row counts of finished collect CTAs; per-row selection
// flags) |
// [rows][words] bitmaps of the keys above the threshold bin | [rows][kCandCap]
// candidates (key, position) | per-segment counts and selection offsets.  The
// first three are zeroed before each use.
struct TkLayout {
  uint32_t* hist;
  uint32_t* ncand;
  uint32_t* ctrl;
  uint32_t* row_done;  // per row: collect CTAs finished (the last one selects)
  uint32_t* sel_done;  // per row: 1 once the row's selection is written (decode step)
  uint32_t* scan_done; // scan CTAs finished (decode step)
  int* scan_pool;      // the scan's tile pool: chunks claimed so far (decode step)
  uint32_t* selready;  // per row: 1 once segoff and the marked bitmap are final, 2 once idx is (decode step)
  uint32_t* bitmap;
  uint2* cand;
  uint32_t* segcnt;    // [rows][kMaxSeg]: keys above the threshold bin per collect segment
  uint32_t* segoff;    // [rows][kMaxSeg + 1]: first selection entry of each segment, then keff
  int64_t words;
};

__host__ __device__ inline size_t tk_ctrl_bytes(int32_t rows) {
  return al256((static_cast<size_t>(kCtrlInts) + 5 * static_cast<size_t>(rows)) * 4);
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
  L.row_done = L.ctrl + kCtrlInts + 2 * rows;
  L.sel_done = L.ctrl + kCtrlInts + 3 * rows;
  L.scan_done = L.ctrl + 1;
  L.scan_pool = reinterpret_cast<int*>(L.ctrl + 2);
  L.selready = L.ctrl + kCtrlInts + 4 * rows;
  b += tk_ctrl_bytes(rows);
  L.bitmap = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * L.words * 4);
  L.cand = reinterpret_cast<uint2*>(b);
  b += al256(static_cast<size_t>(rows) * kCandCap * 8);
  L.segcnt = reinterpret_cast<uint32_t*>(b);
  b += al256(static_cast<size_t>(rows) * kMaxSeg * 4);
  L.segoff = reinterpret_cast<uint32_t*>(b);
  return L;
}

__host__ __device__ inline size_t tk_ws_bytes(int32_t rows, int64_t n_cols) {
  const size_t R = static_cast<size_t>(rows);
  return tk_zero_bytes(rows) + al256(R * ((n_cols + 31) / 32) * 4) + al256(R * kCandCap * 8) +
         al256(R * kMaxSeg * 4) + al256(R * (kMaxSeg + 1) * 4);
}

// Shared scratch of the bodies (static in the standalone kernels, carved from
// dynamic shared memory in the fused step).
struct __align__(16) TkScratch {  // h is read as 16-byte words (the cluster top-k's remote counts)
  int warp_sums[32];
  int s_bin;
  uint32_t s_rank;
  uint32_t s_base;
  uint32_t s_keff;
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

// The NB/NT consecutive bins of thread t from a row's histogram (16-byte
// aligned), as 16-byte loads: scalar loads NB/NT words apart would touch one
// cache line per thread and instruction.
template <int NT, int NB>
__device__ __forceinline__ void tk_load_bins(const uint32_t* hist, int t, uint32_t (&v)[NB / NT]) {
  constexpr int PER = NB / NT;
  static_assert(PER % 4 == 0, "bins per thread");
  const uint4* src = reinterpret_cast<const uint4*>(hist + t * PER);
#pragma unroll
  for (int q = 0; q < PER / 4; ++q) {
    const uint4 x = __ldcg(src + q);
    v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
  }
}

// Bit j of the low byte of x moved to bit 4j.
__device__ __forceinline__ uint32_t spread8(uint32_t x) {
  x &= 0xffu;
  x = (x | (x << 12)) & 0x000f000fu;
  x = (x | (x << 6)) & 0x03030303u;
  x = (x | (x << 3)) & 0x11111111u;
  return x;
}

// One round's scores of a thread: warp w covers the 1024 positions from
// base + 1024 w, lane l and step v the four at base + 1024 w + 128 v + 4 l, so
// every load instruction of the warp reads 512 consecutive bytes.  Only the
// 16-byte groups holding a position below `lim` (the row's length rounded up
// to 4, at most ld, so inside the row) are read; positions at or past the
// row's length are masked when the keys are formed.
struct ColRound {
  float4 x[8];
};

__device__ __forceinline__ void tk_round_load(const float* row, int base, int lim, ColRound& R) {
  const int p0 = base + (threadIdx.x >> 5) * 1024 + (threadIdx.x & 31) * 4;
#pragma unroll
  for (int v = 0; v < 8; ++v) {
    const int p = p0 + v * 128;
    // coherent: the fused step writes the scores in the same launch
    R.x[v] = p < lim ? __ldcg(reinterpret_cast<const float4*>(row + p))
                     : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
  }
}

// The collect pass for segment `seg` of row r: threshold bin b1 of the row from
// its first-digit histogram, then per round of kColRound positions the keys
// above b1 become bitmap words (built from warp ballots, one coalesced store per
// warp) and the keys inside b1 are appended to the row's candidates (one atomic
// per CTA and round).  The first round's scores are requested before the
// histogram is read, and each next round's before this round's atomic.
// Segments are multiples of kColRound positions and cover [0, n_cols), so every
// bitmap word is written.  With count_above, the segment's count of keys above
// b1 goes to segcnt (a split select's offsets); S keeps keff, b1 and the rank
// wanted in b1.  Returns false for an
// empty segment (S then holds nothing of the row).
template <int ID>
__device__ bool tk_collect_cta(const TopkArgs& a, int64_t seg_len, int seg, int r, TkScratch& S,
                               bool count_above = false) {
  constexpr int NT = kCollectThreads;
  static_assert(NT * kWordElems == kColRound && kColRound == (NT / 32) * 1024, "collect round shape");
  static_assert(kMaxBitmapCols <= (1 << 30), "positions fit 32 bits");
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int n = static_cast<int>(a.n_cols);
  if (a.valid_len) {
    const int64_t v = __ldg(a.valid_len + r);
    n = v < 0 ? 0 : (v < n ? static_cast<int>(v) : n);
  }
  const int s0 = seg * static_cast<int>(seg_len);
  const int s1 = s0 + static_cast<int>(seg_len) < static_cast<int>(a.n_cols) ? s0 + static_cast<int>(seg_len)
                                                                              : static_cast<int>(a.n_cols);
  if (s0 >= s1) {
    if (threadIdx.x == 0 && seg < kMaxSeg) tk_layout(a.ws, a.rows, a.n_cols).segcnt[r * kMaxSeg + seg] = 0;
    return false;
  }
  const int lim = ((n + 3) & ~3) < a.ld ? ((n + 3) & ~3) : static_cast<int>(a.ld);
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  ColRound cur;
  tk_round_load(row, s0, lim, cur);
  const TkLayout L = tk_layout(a.ws, a.rows, a.n_cols);
  const uint32_t* hist = L.hist + static_cast<int64_t>(r) * kB1;
  uint32_t hv[kB1 / NT];
  tk_load_bins<NT, kB1>(hist, threadIdx.x, hv);
  const uint32_t total = tk_find<NT, ID, kB1>(hv, static_cast<uint32_t>(a.k), S, true);
  const uint32_t keff = total < static_cast<uint32_t>(a.k) ? total : static_cast<uint32_t>(a.k);
  const uint32_t b1 = keff > 0 ? static_cast<uint32_t>(S.s_bin) : 0xffffffffu;  // none: no bin qualifies
  if (threadIdx.x == 0) S.s_keff = keff;  // with S.s_bin and S.s_rank: the row's threshold bin and rank in it
  uint32_t* bitmap = L.bitmap + static_cast<int64_t>(r) * L.words;
  uint2* cand = L.cand + static_cast<int64_t>(r) * kCandCap;
  int above = 0;  // this thread's keys above the threshold bin
#pragma unroll 1
  for (int base = s0; base < s1; base += kColRound) {
    const int p0 = base + warp * 1024 + lane * 4;
    uint32_t key[8][4];
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int p = p0 + v * 128;
      key[v][0] = p < n ? order_key(cur.x[v].x) : 0u;
      key[v][1] = p + 1 < n ? order_key(cur.x[v].y) : 0u;
      key[v][2] = p + 2 < n ? order_key(cur.x[v].z) : 0u;
      key[v][3] = p + 3 < n ? order_key(cur.x[v].w) : 0u;
    }
    if (base + kColRound < s1) tk_round_load(row, base + kColRound, lim, cur);
    // bitmap word of lane l: positions 32 l .. 32 l + 31 of the warp's 1024,
    // i.e. step v = l / 4, lanes 8 (l % 4) .. 8 (l % 4) + 7
    uint32_t bal[4] = {0u, 0u, 0u, 0u};  // the ballots of step lane / 4
    int nc = 0;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t k = key[v][c];
        const uint32_t bin = k >> 20;
        const uint32_t b = __ballot_sync(0xffffffffu, k != 0u && bin > b1);
        bal[c] = (lane >> 2) == v ? b : bal[c];
        nc += (k != 0u && bin == b1) ? 1 : 0;
      }
    }
    const int sh = 8 * (lane & 3);
    const uint32_t word = spread8(bal[0] >> sh) | (spread8(bal[1] >> sh) << 1) | (spread8(bal[2] >> sh) << 2) |
                          (spread8(bal[3] >> sh) << 3);
    const int wi = (base + warp * 1024) / kWordElems + lane;
    if (wi < L.words) bitmap[wi] = word;
    above += __popc(word);
    int tot;
    const int off = tk_excl_scan<NT, ID>(nc, S.warp_sums, &tot);
    if (threadIdx.x == 0) S.s_base = tot ? atomicAdd(L.ncand + r, static_cast<uint32_t>(tot)) : 0u;
    tk_sync<NT, ID>();
    uint32_t o = S.s_base + static_cast<uint32_t>(off);
    tk_sync<NT, ID>();
    if (nc) {
#pragma unroll
      for (int v = 0; v < 8; ++v) {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const uint32_t k = key[v][c];
          if (k != 0u && (k >> 20) == b1) {
            if (o < static_cast<uint32_t>(kCandCap))
              cand[o] = make_uint2(k, static_cast<uint32_t>(p0 + v * 128 + c));
            ++o;
          }
        }
      }
    }
  }
  if (count_above) {  // the segment's keys above the threshold bin
    int above_tot;
    tk_excl_scan<NT, ID>(above, S.warp_sums, &above_tot);
    if (threadIdx.x == 0 && seg < kMaxSeg) L.segcnt[r * kMaxSeg + seg] = static_cast<uint32_t>(above_tot);
  }
  return true;
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

// Bitmaps of the select body in shared memory: thread t owns the `per`
// consecutive words from t * per and keeps them at t * stride, stride = per | 1
// (odd), so the threads' walks over their own words hit distinct banks.
struct TkPad {
  int per, stride;
};

__host__ __device__ inline TkPad tk_pad(int64_t n_cols, int nt) {
  TkPad p;
  const int64_t words = (n_cols + 31) / 32;
  p.per = static_cast<int>((words + nt - 1) / nt);
  p.stride = p.per | 1;
  return p;
}

// Shared memory of the select body besides TkScratch: two padded bitmaps and
// the candidates.
__host__ __device__ inline size_t tk_final_smem(int64_t n_cols, int nt) {
  const TkPad p = tk_pad(n_cols, nt);
  const size_t bm_words = static_cast<size_t>(nt) * p.stride;
  return 2 * ((bm_words + 1) / 2 * 2) * 4 + static_cast<size_t>(kCandCap) * 8;
}

// Radix select on key bits [19:10] then [9:0] among the keys of bin b1: the
// key T of the rank1-th largest key of the bin, and how many keys equal to T
// (`ties`, the lowest positions first) are still wanted.  The keys are the
// candidates cs[0, nc), or with `overflow` the row's scores (n of them).
template <int NT, int ID>
__device__ void tk_radix_T(const uint2* cs, int nc, bool overflow, const float* row, int64_t n, uint32_t b1,
                           uint32_t rank1, TkScratch& S, uint32_t* T_out, uint32_t* ties_out) {
  const int t = threadIdx.x % NT;
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
  *T_out = T;
  *ties_out = ties;
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
  const TkPad pad = tk_pad(a.n_cols, NT);
  const int bm_words = (NT * pad.stride + 1) / 2 * 2;  // even: keeps cs 8-byte aligned
  uint32_t* bm = fsm;                // selected positions (padded)
  uint32_t* tb = fsm + bm_words;     // positions equal to the threshold key (padded)
  uint2* cs = reinterpret_cast<uint2*>(fsm + 2 * bm_words);
  const DivU32 dper = make_divu32(static_cast<uint32_t>(pad.per));
  auto pw = [&](uint32_t w) -> int {  // padded index of word w
    const uint32_t q = divu32(dper, w);
    return static_cast<int>(q * pad.stride + (w - q * pad.per));
  };
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
  tk_load_bins<NT, kB1>(hist, t, hv);
  const uint32_t n_cand = __ldcg(L.ncand + r);
  const uint32_t* gbm = L.bitmap + static_cast<int64_t>(r) * nwords;
  // eight loads in flight per thread and pass, stored once they have landed
  for (int w0 = t; w0 < nwords; w0 += 8 * NT) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = w0 + u * NT < nwords ? __ldcg(gbm + w0 + u * NT) : 0u;
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      if (w0 + u * NT >= nwords) break;
      const int pi = pw(static_cast<uint32_t>(w0 + u * NT));
      bm[pi] = v[u];
      tb[pi] = 0;
    }
  }
  const bool overflow = n_cand > static_cast<uint32_t>(kCandCap);
  const int nc = overflow ? 0 : static_cast<int>(n_cand);
  for (int c0 = t; c0 < nc; c0 += 4 * NT) {
    uint2 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u] = c0 + u * NT < nc ? __ldcg(L.cand + static_cast<int64_t>(r) * kCandCap + c0 + u * NT) : make_uint2(0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c0 + u * NT < nc) cs[c0 + u * NT] = v[u];
  }
  // keff and the threshold bin
  const uint32_t total = tk_find<NT, ID, kB1>(hv, static_cast<uint32_t>(a.k), S, true);
  const uint32_t keff = total < static_cast<uint32_t>(a.k) ? total : static_cast<uint32_t>(a.k);
  const uint32_t b1 = static_cast<uint32_t>(S.s_bin);
  const uint32_t rank1 = S.s_rank;  // wanted rank inside bin b1
  for (int i = static_cast<int>(keff) + t; i < a.k; i += NT) out[i] = -1;
  if (keff == 0) return;
  // radix select on bits [19:10] then [9:0] among the keys of bin b1
  uint32_t T = 0, ties = 0;
  tk_radix_T<NT, ID>(cs, nc, overflow, row, n, b1, rank1, S, &T, &ties);
  // mark keys of bin b1 above T, and collect the keys equal to T
  if (!overflow) {
    for (int c = t; c < nc; c += NT) {
      const uint2 e = cs[c];
      if (e.x > T) atomicOr(&bm[pw(e.y >> 5)], 1u << (e.y & 31));
      else if (e.x == T) atomicOr(&tb[pw(e.y >> 5)], 1u << (e.y & 31));
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
        if (key > T) atomicOr(&bm[pw(q >> 5)], 1u << (q & 31));
        else if (key == T) atomicOr(&tb[pw(q >> 5)], 1u << (q & 31));
      }
    }
  }
  tk_sync<NT, ID>();
  // ordered compaction: the lowest `ties` positions equal to T join the
  // selection, then the selected positions are written in ascending order;
  // thread t walks its own words (padded: no bank conflicts).
  const int w0 = t * pad.per;
  const int nmine = static_cast<int>(nwords) - w0 < pad.per ? static_cast<int>(nwords) - w0 : pad.per;
  const int pb = t * pad.stride;
  int my_ties = 0;
  for (int i = 0; i < nmine; ++i) my_ties += __popc(tb[pb + i]);
  int tie_tot;
  int tie_before = tk_excl_scan<NT, ID>(my_ties, S.warp_sums, &tie_tot);
  int my_sel = 0;
  for (int i = 0; i < nmine; ++i) {
    const uint32_t x = tb[pb + i];
    const int px = __popc(x);
    const int take = static_cast<int>(ties) - tie_before;
    uint32_t add = 0;
    if (take > 0) add = take >= px ? x : low_bits(x, take);
    tie_before += px;
    const uint32_t merged = bm[pb + i] | add;
    bm[pb + i] = merged;
    my_sel += __popc(merged);
  }
  int sel_tot;
  int o = tk_excl_scan<NT, ID>(my_sel, S.warp_sums, &sel_tot);
  // The positions are gathered in shared memory (the candidates' space, free
  // now) and written out coalesced: written straight from the walk, every
  // store instruction of a warp would touch up to 32 lines.
  int32_t* os = reinterpret_cast<int32_t*>(cs);
  const bool staged = a.k <= 2 * kCandCap;
  for (int i = 0; i < nmine; ++i) {
    uint32_t x = bm[pb + i];
    while (x) {
      const int b = __ffs(x) - 1;
      x &= x - 1;
      if (o < a.k) {
        if (staged) os[o] = (w0 + i) * 32 + b;
        else out[o] = (w0 + i) * 32 + b;
      } else {
        record_error(a.status, LSA_ERR_BOUNDS, r, o);  // cannot happen
      }
      ++o;
    }
  }
  if (staged) {
    tk_sync<NT, ID>();
    const int n_out = static_cast<int>(keff);
    for (int i = t; i < n_out; i += NT) out[i] = os[i];
  }
  tk_sync<NT, ID>();  // shared memory free for the caller's next use
}

// Split select of row r, run by the row's last collect CTA in a decode step
// (NT threads; fsm: shared memory of at least tk_split_smem() bytes, 8-byte
// aligned).  Instead of compacting the row's selection it makes the row's
// bitmap exact (marks the threshold bin's keys above T and the `ties` lowest
// positions equal to T) and stores, per collect segment, the first selection
// entry it holds (segoff[r][s], then keff at [nseg]): a consumer of entries
// [e0, e1) then compacts only the segments those entries fall in.  Returns
// false, having changed nothing a full select relies on, when the candidates
// overflowed their list or more than kTieCap keys equal T; the caller then
// runs the full select.
__host__ __device__ inline size_t tk_split_smem() {
  return (static_cast<size_t>(kMaxSeg) + kTieCap + 8) * 4 + static_cast<size_t>(kCandCap) * 8;
}

template <int NT, int ID>
__device__ bool tk_split_select(const TopkArgs& a, int r, int nseg, int64_t seg_len, uint32_t keff, uint32_t b1,
                                uint32_t rank1, uint32_t* fsm, TkScratch& S) {
  const int t = threadIdx.x % NT;
  const TkLayout L = tk_layout(a.ws, a.rows, a.n_cols);
  uint32_t* seg_add = fsm;                              // [kMaxSeg]
  uint32_t* eqpos = fsm + kMaxSeg;                      // [kTieCap]
  uint32_t* s_eq = fsm + kMaxSeg + kTieCap;             // count of keys equal to T
  uint2* cs = reinterpret_cast<uint2*>(fsm + kMaxSeg + kTieCap + 8);
  uint32_t* segoff = L.segoff + static_cast<int64_t>(r) * (kMaxSeg + 1);
  if (keff == 0) {
    for (int i = t; i <= nseg; i += NT) segoff[i] = 0;
    return true;
  }
  const uint32_t n_cand = __ldcg(L.ncand + r);
  if (n_cand > static_cast<uint32_t>(kCandCap)) return false;
  const int nc = static_cast<int>(n_cand);
  for (int c0 = t; c0 < nc; c0 += 4 * NT) {
    uint2 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      v[u] = c0 + u * NT < nc ? __ldcg(L.cand + static_cast<int64_t>(r) * kCandCap + c0 + u * NT) : make_uint2(0, 0);
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (c0 + u * NT < nc) cs[c0 + u * NT] = v[u];
  }
  for (int i = t; i < kMaxSeg; i += NT) seg_add[i] = 0;
  if (t == 0) *s_eq = 0;
  uint32_t T, ties;
  tk_radix_T<NT, ID>(cs, nc, false, nullptr, 0, b1, rank1, S, &T, &ties);  // its barriers publish the above
  // keys equal to T: their positions, to rank (ties are broken by lowest position)
  for (int c = t; c < nc; c += NT) {
    if (cs[c].x == T) {
      const uint32_t i = atomicAdd(s_eq, 1u);
      if (i < static_cast<uint32_t>(kTieCap)) eqpos[i] = cs[c].y;
    }
  }
  tk_sync<NT, ID>();
  const int n_eq = static_cast<int>(*s_eq);
  if (n_eq > kTieCap) return false;  // nothing marked yet
  uint32_t* bitmap = L.bitmap + static_cast<int64_t>(r) * L.words;
  for (int c = t; c < nc; c += NT) {
    const uint2 e = cs[c];
    if (e.x > T) {
      atomicOr(bitmap + (e.y >> 5), 1u << (e.y & 31));
      atomicAdd(seg_add + e.y / static_cast<uint32_t>(seg_len), 1u);
    }
  }
  for (int i = t; i < n_eq; i += NT) {
    const uint32_t p = eqpos[i];
    int rank = 0;
    for (int j = 0; j < n_eq; ++j) rank += eqpos[j] < p ? 1 : 0;
    if (rank < static_cast<int>(ties)) {
      atomicOr(bitmap + (p >> 5), 1u << (p & 31));
      atomicAdd(seg_add + p / static_cast<uint32_t>(seg_len), 1u);
    }
  }
  tk_sync<NT, ID>();
  // first entry of each segment: keys above the bin plus the marked ones, scanned
  const uint32_t mine = t < nseg ? __ldcg(L.segcnt + r * kMaxSeg + t) + seg_add[t] : 0u;
  int total;
  const int before = tk_excl_scan<NT, ID>(static_cast<int>(mine), S.warp_sums, &total);
  if (t < nseg) segoff[t] = static_cast<uint32_t>(before);
  if (t == 0) segoff[nseg] = static_cast<uint32_t>(total);
  if (t == 0 && total != static_cast<int>(keff)) record_error(a.status, LSA_ERR_BOUNDS, r, total);  // cannot happen
  return true;
}

}  // namespace tk
}  // namespace lsa
