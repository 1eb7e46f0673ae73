#pragma once
// Lightning-indexer scan on the sm_100a tensor cores: the device code of one
// CTA, shared by the standalone scan kernel and the fused decode step.
//
// Before each DSA layer the lightning indexer scores every cached token of the
// sequence, and at long context this scan is where decode time goes (MLI
// "Multi-layer Indexer" abstract, sentences 2-3).  Score of token s for a query
// row: I(s) = sum_h w[h] * ReLU(q[h] . K[s]) over 64 indexer heads of dim 128
// (DSA lightning indexer, DeepSeek-V3.2-Exp report); FP8 keys carry a per-token
// scale (the compact indexer keys of the LeanSparse episode page).
//
// Mapping: keys are the MMA's M side (128 tokens per tile, one TMEM lane per
// token) and the query heads its N side, so after the MMA every epilogue thread
// owns one token with all of its head dot products in TMEM; the ReLU-weighted
// head reduction then runs in registers.  Decode groups one query row per tile
// (N = 64); the causal prefill groups 4 rows of one sequence (N = 256), reusing
// each key tile 4 times.  FP8 keys go straight to kind::f8f6f4 MMAs: the bf16
// query is split into two e4m3 terms (hi + lo, per-head power-of-two scale
// folded into w; exact for entries within 2^10 of the head's largest, see
// stage_query_fp8), so no key conversion is needed: the decode accumulates
// both terms into one column per head (twice the K-steps), the prefill keeps
// them as separate columns (twice the N).
//
// One persistent CTA per SM, warp-specialised:
//   warp 0  TMA producer: 64-row boxes of the key cache (block-table gather)
//   warp 1  MMA issuer of the even tiles (one thread) + TMEM owner
//   warp 2  query staging: query rows -> swizzled smem operand, weights
//   warps 3-6 epilogue: TMEM -> registers, ReLU-weighted sum, score stores
//            (warps 3-10 with two epilogue groups)
//   last    MMA issuer of the odd tiles (one thread)
// Two issuers, one per accumulator: an MMA of this size occupies the tensor
// pipe for about as long as its issuer spends on the waits and bookkeeping of
// a tile, so with one issuer the pipe idled half of the time.
// Work: the query rows' tiles in row order, each CTA an even contiguous
// share; every role walks the same sequence.  Optionally (decode) the CTAs
// share only part of it and claim the rest in chunks from a counter, the
// producer publishing each chunk to the other roles through a ring.
// Every wait is bounded; a timeout records LSA_ERR_TIMEOUT and unwinds.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace lsa {
namespace scan {

constexpr int kHeads = 64;       // indexer heads
constexpr int kDim = 128;        // indexer head dim
constexpr int kTile = 128;       // tokens per tile (MMA M, TMEM lanes)
constexpr int kBoxRows = 64;     // rows per TMA box (one 64-token page or half tile)
constexpr int kBoxX = 32;        // 4-byte TMA elements per 128-byte K block
constexpr int kScaleBox = 68;    // FP8 scales per box load: 64 + up to 3 for the 16-byte aligned start
constexpr int kScaleSlot = 96;   // floats per scale slot: a TMA destination starts on a 128-byte boundary
constexpr int kThreads = 256;    // 8 warps (one epilogue group)
// Threads of a scan CTA with EG epilogue groups of 4 warps (warps 3.., the
// groups taking alternate tiles), the second MMA issuer's warp last.
template <int EG>
constexpr int scan_threads() { return kThreads + (EG - 1) * 128; }
template <int EG>
constexpr int warp_mma2() { return 3 + 4 * EG; }
constexpr int kWarpProd = 0, kWarpMma = 1, kWarpQ = 2, kWarpEpi = 3;
constexpr int kSmemLimit = 232448;
constexpr int kBarrierId = 1;    // named barrier of the scan's threads (a fused block holds more threads)
// Pooled schedule (decode): tiles claimed from a global counter reach the
// other roles as segments through a ring of kRing slots; a pooled launch has
// at most kPoolRows query rows (the planner's one row per thread).
constexpr int kRing = 8;
constexpr int kSlotInts = 8;     // r0, j0, n, b, tiles, vis (2 ints), spare
constexpr int kPoolRows = kThreads;

template <int NTH = kThreads>
__device__ __forceinline__ void scan_sync() {
  asm volatile("bar.sync %0, %1;" ::"n"(kBarrierId), "n"(NTH) : "memory");
}

template <int KDT, int QB, bool GATHER = false>
struct Cfg {
  static constexpr bool kFp8 = KDT == LSA_FP8_E4M3;
  static constexpr int kN = (kFp8 ? 2 * kHeads : kHeads) * QB;    // query operand rows
  static constexpr int kKBlocks = kFp8 ? 1 : 2;                    // 128-byte K blocks per row
  static constexpr int kKBlockBytes = kTile * 128;                 // A: 128 rows x 128 B
  static constexpr int kTileBytes = kKBlocks * kKBlockBytes;
  static constexpr int kBoxBytes = kBoxRows * 128;
  static constexpr int kQKBlockBytes = kN * 128;                   // B: N rows x 128 B per K block
  static constexpr int kQBytes = kKBlocks * kQKBlockBytes;
  // query operand buffers: decode stages the next group's (or segment's)
  // query while the MMAs of the current one run
  static constexpr int kNQ = QB == 1 ? 2 : 1;
  static constexpr int kWBytes = QB * kHeads * 4;
  static constexpr int kHistBytes = QB == 1 ? kTopkBins1 * 4 : 0;  // fused first top-k histogram (decode)
  // Per stage besides the keys: the key rows of its two boxes (written by the
  // producer for the epilogue) and, for FP8, the two boxes' scales (TMA).
  // Gathered candidates: the stage's masks of rows with a key (4 words) and of
  // rows whose position or block was out of range (4 words).
  static constexpr int kMetaBytes = 2 * 4 + (kFp8 ? 2 * kScaleSlot * 4 : 0) + (GATHER ? 8 * 4 : 0);
  static constexpr int kRawBytes = kFp8 ? QB * kHeads * kDim * 2 : 0;  // FP8: bf16 query rows before the split
  // pooled schedule (decode, TMA producer): the ring's barriers and slots and
  // the rows' first tiles and visible positions
  static constexpr bool kPool = QB == 1 && !GATHER;
  static constexpr int kPoolBytes = kPool ? kRing * (2 * 8 + kSlotInts * 4) + 2 * kPoolRows * 4 : 0;
  static constexpr int kFixed = kNQ * kQBytes + kNQ * kWBytes + kRawBytes + kHistBytes + 640 /*barriers, scratch*/ +
                                kPoolBytes + 1024 /*align*/;
  static constexpr int kNSmax = (kSmemLimit - kFixed) / (kTileBytes + kMetaBytes);
  static constexpr int kNS = kNSmax > 12 ? 12 : kNSmax;            // key stages
  // FP8 decode: the query's hi and lo terms (rows 0-63 and 64-127 of the
  // query operand) accumulate into the same 64 columns, one per head, as
  // K-steps 5-8 over the same key tile: the epilogue reads half the columns.
  static constexpr bool kCat = kFp8 && QB == 1;
  static constexpr int kNmma = kCat ? kHeads : kN;                 // MMA N
  static constexpr int kAccCols = kNmma;
  // Accumulators in TMEM, used round robin: an accumulator's turn spans its
  // MMAs, the commit's arrival, the epilogue's reads and the release back to
  // the issuer, so four (where they fit) keep the MMAs of a tile from waiting
  // for the epilogue of the tile two before it.
  static constexpr int kAcc = 4 * kAccCols <= 512 ? 4 : 2;
  static constexpr int kTmemCols = kAcc * kAccCols <= 32 ? 32 : kAcc * kAccCols <= 64 ? 64
                                   : kAcc * kAccCols <= 128 ? 128 : kAcc * kAccCols <= 256 ? 256 : 512;
  static constexpr int kSmemBytes = kNS * (kTileBytes + kMetaBytes) + kFixed;
  static constexpr uint32_t kIdesc = tc::idesc(kFp8 ? tc::kFmtE4M3 : tc::kFmtBF16,
                                               kFp8 ? tc::kFmtE4M3 : tc::kFmtBF16, kTile, kNmma);
  static_assert(kNS >= 3, "too few key stages");
  static_assert(2 * kN <= 512, "accumulators exceed TMEM");
  static_assert(kSmemBytes <= kSmemLimit, "shared memory");
  static_assert(!GATHER || (KDT == LSA_BF16 && QB == 1), "candidate gather: bf16 keys, one row per tile");
};

// Stages of the configurations that run: decode 5 (bf16) and 9 (FP8) tiles in
// flight, the causal prefill 5 (bf16, 4 rows per tile) and 9 (FP8, 2 rows).
static_assert(Cfg<LSA_BF16, 1>::kNS == 5 && Cfg<LSA_FP8_E4M3, 1>::kNS == 9, "decode stages");
static_assert(Cfg<LSA_BF16, 4>::kNS == 5 && Cfg<LSA_FP8_E4M3, 2>::kNS == 9, "prefill stages");

// ---------------------------------------------------------------- work items

__device__ __forceinline__ int seq_of(const ScoresArgs& a, int r) { return a.row_seq ? __ldg(a.row_seq + r) : r; }

// Visible positions of query row r (0 for an invalid row).
__device__ __forceinline__ int64_t row_visible(const ScoresArgs& a, int r, int* b_out) {
  const int b = seq_of(a, r);
  *b_out = b;
  if (b < 0 || b >= a.cache.batch) return 0;
  int64_t L = __ldg(a.cache.seq_lens + b);
  L = L < 0 ? 0 : (L > a.cache.max_len ? a.cache.max_len : L);
  if (a.row_pos) {
    int64_t p = static_cast<int64_t>(__ldg(a.row_pos + r)) + 1;
    p = p < 0 ? 0 : p;
    L = p < L ? p : L;
  }
  // candidate re-scoring: the row's "positions" are its candidate entries
  if (a.cand) L = L < a.cand_ld ? L : a.cand_ld;
  return L;
}

// Positions of query row r a candidate may name: [0, cap) (the row's visible
// range, before the candidate list shortens it).
__device__ __forceinline__ int64_t row_cap(const ScoresArgs& a, int r, int b) {
  if (b < 0 || b >= a.cache.batch) return 0;
  int64_t L = __ldg(a.cache.seq_lens + b);
  L = L < 0 ? 0 : (L > a.cache.max_len ? a.cache.max_len : L);
  if (a.row_pos) {
    int64_t p = static_cast<int64_t>(__ldg(a.row_pos + r)) + 1;
    p = p < 0 ? 0 : p;
    L = p < L ? p : L;
  }
  return L;
}

// A group is a run of up to QB consecutive query rows of one sequence that
// does not cross a multiple of QB; its rows share every key tile.
template <int QB>
__device__ __forceinline__ bool is_leader(const ScoresArgs& a, int r) {
  if (QB == 1 || r % QB == 0) return true;
  return seq_of(a, r) != seq_of(a, r - 1);
}

struct Group {
  int r0, nrows, b, tiles;
  int64_t vis;  // max visible positions over the group's rows
};

template <int QB>
__device__ Group group_at(const ScoresArgs& a, int r0) {
  Group g;
  g.r0 = r0;
  int b;
  int64_t vis = row_visible(a, r0, &b);
  g.b = b;
  int n = 1;
  if (QB > 1) {
    while (n < QB && r0 + n < a.rows && ((r0 + n) % QB) != 0 && seq_of(a, r0 + n) == b) {
      int bb;
      int64_t v = row_visible(a, r0 + n, &bb);
      vis = v > vis ? v : vis;
      ++n;
    }
  }
  g.nrows = n;
  g.vis = vis;
  g.tiles = static_cast<int>((vis + kTile - 1) / kTile);
  return g;
}

// Walks the CTA's items (group, tile) in global order, skipping empty groups.
template <int QB>
struct Walker {
  Group g;
  int j;
  __device__ void start(const ScoresArgs& a, int r0, int j0) {
    g = group_at<QB>(a, r0);
    j = j0;
  }
  __device__ void start(const Group& g0, int j0) {
    g = g0;
    j = j0;
  }
  __device__ void next(const ScoresArgs& a) {
    if (++j < g.tiles) return;
    j = 0;
    int r = g.r0 + g.nrows;
    while (r < a.rows) {
      g = group_at<QB>(a, r);
      if (g.tiles > 0) return;
      r += g.nrows;
    }
    g.tiles = 0;  // past the end
  }
};

template <int NTH>
__device__ __forceinline__ int block_sum_i64_scan(int64_t v, int64_t* warp_buf, int64_t* incl, int64_t* total) {
  // inclusive scan over the block (NTH threads), returns nothing; used by the planner
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_buf[warp] = x;
  scan_sync<NTH>();
  int64_t before = 0, tot = 0;
  for (int w = 0; w < NTH / 32; ++w) {
    if (w < warp) before += warp_buf[w];
    tot += warp_buf[w];
  }
  *incl = before + x;
  *total = tot;
  scan_sync<NTH>();
  return 0;
}

struct Plan {
  int r_first;  // leader row of the CTA's first item
  int j_first;
  int64_t n_items;
  int64_t pool_lo, pool_hi;  // pooled launch: the tiles claimed from the pool
};

// The tiles [lo, hi) of `tot` that this launch covers (ScoresArgs::split_part).
__device__ __forceinline__ void launch_tiles(const ScoresArgs& a, int64_t tot, int64_t* lo, int64_t* hi) {
  *lo = 0;
  *hi = tot;
  if (a.split_part == 0 || a.split_free <= 0) return;
  // the first part: what split_free CTAs stream while the other SMs are busy
  int64_t first = static_cast<int64_t>(a.split_busy_us / a.split_tile_us) * a.split_free;
  first = first < 0 ? 0 : (first > tot ? tot : first);
  if (a.split_part == 1) *hi = first;
  else *lo = first;
}

// Every thread of the CTA takes part: total tiles, this CTA's share, and the
// group holding its first tile.  A pooled launch (pool_start set: one query
// row per tile, at most kPoolRows rows) splits its first pool_static_pm
// thousandths of the tiles evenly over the CTAs and leaves the rest to the
// pool; pool_start[r] receives row r's first tile in the launch's order and
// pool_start[kPoolRows + r] its visible positions.
template <int QB, int NTH = kThreads>
__device__ Plan plan_work(const ScoresArgs& a, int64_t* sbuf, int* sfound, int* pool_start = nullptr) {
  Plan p;
  p.r_first = 0;
  p.j_first = 0;
  p.pool_lo = p.pool_hi = 0;
  if (a.rows <= NTH) {  // one row per thread: a single block scan
    const int r = threadIdx.x;
    int64_t t = 0, vis = 0;
    if (r < a.rows && is_leader<QB>(a, r)) {
      const Group g = group_at<QB>(a, r);
      t = g.tiles;
      vis = g.vis;
    }
    int64_t incl, tot;
    block_sum_i64_scan<NTH>(t, sbuf, &incl, &tot);
    // this launch's tiles [lo, hi), split evenly over its CTAs
    int64_t lo, hi;
    launch_tiles(a, tot, &lo, &hi);
    if (pool_start) {
      // row r's first tile, then (kPoolRows further on) its visible positions
      if (r < a.rows) {
        pool_start[r] = static_cast<int>(incl - t);
        pool_start[kPoolRows + r] = static_cast<int>(vis);
      }
      lo = 0;
      hi = tot * a.pool_static_pm / 1000;
      p.pool_lo = hi;
      p.pool_hi = tot;
    }
    const int64_t t0 = lo + (hi - lo) * blockIdx.x / gridDim.x;
    p.n_items = lo + (hi - lo) * (blockIdx.x + 1) / gridDim.x - t0;
    if (p.n_items <= 0) return p;
    const int64_t start = incl - t;
    if (t > 0 && start <= t0 && t0 < start + t) {  // exactly one thread holds tile t0
      sfound[0] = r;
      sfound[1] = static_cast<int>(t0 - start);
    }
    scan_sync<NTH>();
    p.r_first = sfound[0];
    p.j_first = sfound[1];
    return p;
  }
  int64_t total = 0;
  for (int base = 0; base < a.rows; base += NTH) {
    const int r = base + threadIdx.x;
    int64_t t = 0;
    if (r < a.rows && is_leader<QB>(a, r)) t = group_at<QB>(a, r).tiles;
    int64_t incl, tot;
    block_sum_i64_scan<NTH>(t, sbuf, &incl, &tot);
    total += tot;
  }
  int64_t lo, hi;
  launch_tiles(a, total, &lo, &hi);
  const int64_t t0 = lo + (hi - lo) * blockIdx.x / gridDim.x;
  const int64_t t1 = lo + (hi - lo) * (blockIdx.x + 1) / gridDim.x;
  p.n_items = t1 - t0;
  if (p.n_items <= 0) return p;
  if (threadIdx.x == 0) sfound[0] = -1;
  scan_sync<NTH>();
  int64_t acc = 0;
  for (int base = 0; base < a.rows; base += NTH) {
    const int r = base + threadIdx.x;
    int64_t t = 0;
    if (r < a.rows && is_leader<QB>(a, r)) t = group_at<QB>(a, r).tiles;
    int64_t incl, tot;
    block_sum_i64_scan<NTH>(t, sbuf, &incl, &tot);
    const int64_t start = acc + incl - t;
    if (t > 0 && start <= t0 && t0 < start + t) {
      sfound[0] = r;
      sfound[1] = static_cast<int>(t0 - start);
    }
    acc += tot;
    scan_sync<NTH>();
    if (sfound[0] >= 0) break;
  }
  p.r_first = sfound[0];
  p.j_first = sfound[1];
  return p;
}

// ---------------------------------------------------------------- query staging

// bf16: B row n = qq * 64 + h holds q[row r0+qq][h][:] in two 128-byte K blocks.
// Every 16-byte piece (and the weights) is a cp.async issued at once, so the
// staging costs one memory round trip even while the key loads crowd the
// memory system; rows of absent queries are zero-filled.
template <int QB>
__device__ void stage_query_bf16(const ScoresArgs& a, const Group& g, uint8_t* qbuf, float* wbuf, int lane) {
  constexpr int N = kHeads * QB;
  const uint8_t* src = reinterpret_cast<const uint8_t*>(a.q_idx);
  for (int idx = lane; idx < N * (kDim / 8); idx += 32) {
    const int n = idx >> 4, c = idx & 15;
    const int qq = n / kHeads, h = n % kHeads;
    const bool live = qq < g.nrows;
    const uint8_t* p = src + ((static_cast<int64_t>(live ? g.r0 + qq : g.r0) * kHeads + h) * kDim) * 2 + c * 16;
    tc::cp_async16_zfill(qbuf + (c >> 3) * (N * 128) + tc::sw128_offset(n, c & 7), p, live ? 16u : 0u);
  }
  for (int i = lane; i < QB * (kHeads / 4); i += 32) {
    const int qq = i / (kHeads / 4), c = i % (kHeads / 4);
    const bool live = qq < g.nrows;
    tc::cp_async16_zfill(wbuf + qq * kHeads + c * 4, a.w + static_cast<int64_t>(live ? g.r0 + qq : g.r0) * kHeads + c * 4,
                         live ? 16u : 0u);
  }
  tc::cp_async_wait_all();
}

__device__ __forceinline__ uint32_t pack_e4m3x4(float a, float b, float c, float d) {
  const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(make_float2(a, b), __NV_SATFINITE, __NV_E4M3);
  const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(make_float2(c, d), __NV_SATFINITE, __NV_E4M3);
  return static_cast<uint32_t>(lo) | (static_cast<uint32_t>(hi) << 16);
}

// fp8: per (query, head) a power-of-two scale s puts max|q| into [224, 448];
// q*s ~ hi + lo with hi = e4m3(q*s), lo = e4m3(q*s - hi).  A bf16 entry has 8
// significant bits and each e4m3 term 4, so the split is exact while both
// terms are normal e4m3 numbers (magnitude >= 2^-6), which holds for
// |q*s| >= 2^-2, i.e. entries at least 2^-10 of the head's largest.  Smaller
// entries are not exact: a term in e4m3's subnormal range is rounded to its
// step 2^-9, an absolute error of at most 2^-10 in scaled units (below 5e-6 of
// the head's largest entry), well inside the 2e-2 score tolerance.  B row
// qq*128 + h holds hi, qq*128 + 64 + h holds lo; w' = w / s.
// The raw rows and the weights arrive by cp.async in one round trip; half a
// warp then converts one head (8 dims per lane) from shared memory.
template <int QB>
__device__ void stage_query_fp8(const ScoresArgs& a, const Group& g, uint8_t* qbuf, float* wbuf, uint8_t* raw,
                                int lane) {
  const uint8_t* src = reinterpret_cast<const uint8_t*>(a.q_idx);
  for (int idx = lane; idx < QB * kHeads * (kDim / 8); idx += 32) {
    const int n = idx >> 4, c = idx & 15;
    const int qq = n / kHeads, h = n % kHeads;
    const bool live = qq < g.nrows;
    const uint8_t* p = src + ((static_cast<int64_t>(live ? g.r0 + qq : g.r0) * kHeads + h) * kDim) * 2 + c * 16;
    tc::cp_async16_zfill(raw + n * (kDim * 2) + c * 16, p, live ? 16u : 0u);
  }
  for (int i = lane; i < QB * (kHeads / 4); i += 32) {
    const int qq = i / (kHeads / 4), c = i % (kHeads / 4);
    const bool live = qq < g.nrows;
    tc::cp_async16_zfill(wbuf + qq * kHeads + c * 4, a.w + static_cast<int64_t>(live ? g.r0 + qq : g.r0) * kHeads + c * 4,
                         live ? 16u : 0u);
  }
  tc::cp_async_wait_all();
  __syncwarp();
  const int half = lane >> 4, seg = lane & 15;  // seg: dims [8 seg, 8 seg + 8)
#pragma unroll 2
  for (int n0 = 0; n0 < QB * kHeads; n0 += 2) {
    const int n = n0 + half;
    const int qq = n / kHeads, h = n % kHeads;
    const uint4 v = *reinterpret_cast<const uint4*>(raw + n * (kDim * 2) + seg * 16);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float x[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = __uint_as_float(wv[j] << 16);
      x[2 * j + 1] = __uint_as_float(wv[j] & 0xffff0000u);
    }
    float mx = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) mx = fmaxf(mx, fabsf(x[j]));
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    // Largest power of two s = 2^k with mx * s <= 448 = 1.75 * 2^8: for
    // mx = m * 2^E (1 <= m < 2), k = 8 - E if m <= 1.75, else 7 - E.
    int k = 0;
    if (mx > 0.f) {
      const uint32_t mb = __float_as_uint(mx);
      const int E = static_cast<int>(mb >> 23) - 127;
      k = (mb & 0x7fffffu) <= 0x600000u ? 8 - E : 7 - E;
      k = k < -126 ? -126 : (k > 126 ? 126 : k);
    }
    const float sc = __uint_as_float(static_cast<uint32_t>(k + 127) << 23);
    const float inv = __uint_as_float(static_cast<uint32_t>(127 - k) << 23);
    uint32_t hw[2], lw[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float xs[4], lv[4];
#pragma unroll
      for (int e4 = 0; e4 < 4; ++e4) xs[e4] = x[4 * u + e4] * sc;
      hw[u] = pack_e4m3x4(xs[0], xs[1], xs[2], xs[3]);
#pragma unroll
      for (int e4 = 0; e4 < 4; ++e4) lv[e4] = xs[e4] - e4m3_to_float(static_cast<uint8_t>(hw[u] >> (8 * e4)));
      lw[u] = pack_e4m3x4(lv[0], lv[1], lv[2], lv[3]);
    }
    const int row_hi = qq * 2 * kHeads + h, row_lo = row_hi + kHeads;
    const uint32_t off = (seg & 1) * 8;
    *reinterpret_cast<uint2*>(qbuf + tc::sw128_offset(row_hi, seg >> 1) + off) = make_uint2(hw[0], hw[1]);
    *reinterpret_cast<uint2*>(qbuf + tc::sw128_offset(row_lo, seg >> 1) + off) = make_uint2(lw[0], lw[1]);
    if (seg == 0) wbuf[n] *= inv;  // w / s, exact for a power of two
  }
}

// ---------------------------------------------------------------- candidate gather

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}

// Producer warp of the candidate re-scoring: each tile's 128 key rows (the
// row's candidate entries j*128 .. j*128+127) are copied with cp.async into
// the stage in the image the TMA boxes give (two 128-byte K blocks, 128-byte
// swizzle); rows without a key are zero-filled.  Each half-warp copies one
// 256-byte row per instruction (coalesced).  The rows of kBatch tiles are
// resolved ahead (candidate entry, then block table) with all of their loads
// in flight, so those latencies are paid once per batch.  A stage is full once
// every lane's copies have landed (one cp.async arrival per lane) and lane 0
// has published the stage's masks: rows with a key, and rows whose position
// or block was out of range (their scores become NaN; the first is reported).
template <class C>
__device__ void gather_producer(const ScoresArgs& a, const Plan& plan, const CacheAddr& ad, uint8_t* stages,
                                uint32_t* smask, uint64_t* full, uint64_t* empty, volatile int* abort_flag,
                                int lane) {
  if (plan.n_items <= 0) return;
  constexpr int kBatch = 4;
  constexpr int kRowBytes = kDim * 2;
  const uint8_t* keys = static_cast<const uint8_t*>(a.cache.idx_keys);
  Walker<1> W;
  W.start(a, plan.r_first, plan.j_first);
  int64_t it = 0;
  bool failed = false;
  while (it < plan.n_items && !failed) {
    const int nb = plan.n_items - it < kBatch ? static_cast<int>(plan.n_items - it) : kBatch;
    int32_t pos[kBatch][4];
    int rb[kBatch], rr[kBatch];
    int64_t cap[kBatch];
    {
      Walker<1> Wu = W;
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        rb[u] = -1;
        rr[u] = 0;
        cap[u] = 0;
#pragma unroll
        for (int m = 0; m < 4; ++m) pos[u][m] = -1;
        if (u < nb) {
          rr[u] = Wu.g.r0;
          rb[u] = Wu.g.b;
          cap[u] = row_cap(a, Wu.g.r0, Wu.g.b);
          const int32_t* cl = a.cand + static_cast<int64_t>(Wu.g.r0) * a.cand_ld;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const int64_t slot = static_cast<int64_t>(Wu.j) * kTile + lane + 32 * m;
            if (slot < Wu.g.vis) pos[u][m] = __ldg(cl + slot);
          }
          Wu.next(a);
        }
      }
      W = Wu;
    }
    // key rows: >= 0 a row, -3 no candidate (padding), -1 out of range
    int32_t row[kBatch][4];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int32_t p = pos[u][m];
        int32_t rw = -3;
        if (p >= 0) {
          rw = -1;
          if (p < cap[u]) {
            if (ad.block_size == 0) {
              rw = static_cast<int32_t>(static_cast<int64_t>(rb[u]) * ad.max_len + p);
            } else {
              const int64_t lb = p / ad.block_size;
              if (lb < ad.max_blocks) {
                const int32_t blk = __ldg(ad.block_table + static_cast<int64_t>(rb[u]) * ad.max_blocks + lb);
                if (blk >= 0 && blk < ad.n_blocks)
                  rw = static_cast<int32_t>(static_cast<int64_t>(blk) * ad.block_size + (p - lb * ad.block_size));
              }
            }
          }
          if (rw == -1) record_error(a.status, LSA_ERR_BOUNDS, rr[u], p);
        }
        row[u][m] = rw;
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (u >= nb) break;
      const int s = static_cast<int>(it % C::kNS);
      const uint32_t ph = static_cast<uint32_t>((it / C::kNS) & 1);
      // lane 0 waits for the stage; the verdict is broadcast so the warp stays converged
      bool ok = true;
      if (lane == 0) ok = tc::mbar_wait(&empty[s], ph ^ 1, abort_flag);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) {
          record_error(a.status, LSA_ERR_TIMEOUT, 0, 9);
          *abort_flag = 1;
        }
        failed = true;
        break;
      }
      __syncwarp();
      uint32_t have[4], bad[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        have[m] = __ballot_sync(0xffffffffu, row[u][m] >= 0);
        bad[m] = __ballot_sync(0xffffffffu, row[u][m] == -1);
      }
      uint8_t* st = stages + s * C::kTileBytes;
      const int c = lane & 15;  // 16-byte chunk of the row (K block c >> 3)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
#pragma unroll 4
        for (int i2 = 0; i2 < 16; ++i2) {
          const int src = 2 * i2 + (lane >> 4);
          const int32_t rv = __shfl_sync(0xffffffffu, row[u][m], src);
          const uint32_t ri = static_cast<uint32_t>(32 * m + src);
          const uint8_t* g = keys + static_cast<int64_t>(rv >= 0 ? rv : 0) * kRowBytes + c * 16;
          tc::cp_async16_zfill(st + (c >> 3) * C::kKBlockBytes + tc::sw128_offset(ri, static_cast<uint32_t>(c & 7)), g,
                               rv >= 0 ? 16u : 0u);
        }
      }
      uint64_t* fb = &full[it % (2 * C::kNS)];  // the item's full barrier (see scan_cta)
      cp_async_arrive_noinc(fb);
      if (lane == 0) {
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          smask[8 * s + m] = have[m];
          smask[8 * s + 4 + m] = bad[m];
        }
        tc::mbar_arrive(fb);  // release: the masks are visible to the epilogue's acquire
      }
      ++it;
    }
    failed = __shfl_sync(0xffffffffu, failed || *abort_flag, 0);
  }
  // every copy must land before the CTA's shared memory is released
  tc::cp_async_wait_all();
}

// ---------------------------------------------------------------- the kernel

// One CTA's share of the scan, run by threads [0, kThreads) of the block
// (the only threads that take part in its barriers).  `tmem_slot` holds (or,
// once the first barrier of the plan has passed, will hold) the base of at
// least Cfg::kTmemCols allocated TMEM columns.  Every mbarrier it used is
// invalidated before it returns, so the caller may reuse the shared memory.
template <int KDT, int QB, bool GATHER = false, int EG = 1>
__device__ __forceinline__ void scan_cta(const CUtensorMap* tmap_p, const CUtensorMap* smap_p, const ScoresArgs& a,
                                         uint8_t* smem_raw, const volatile uint32_t* tmem_slot) {
  using C = Cfg<KDT, QB, GATHER>;
  constexpr int NTH = scan_threads<EG>();
  static_assert(EG == 1 || EG == 2, "one or two epilogue groups");
  const CUtensorMap& tmap = *tmap_p;
  const CUtensorMap& smap = *smap_p;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  // Offsets keep every TMA destination 128-byte and every cp.async one 16-byte aligned.
  uint8_t* qbufs = stages + C::kNS * C::kTileBytes;                                  // 1024-aligned operands
  float* wbufs = reinterpret_cast<float*>(qbufs + C::kNQ * C::kQBytes);
  uint8_t* qraw = reinterpret_cast<uint8_t*>(wbufs) + C::kNQ * C::kWBytes;          // FP8: raw query rows
  float* sscale = reinterpret_cast<float*>(qraw + C::kRawBytes);                     // FP8: [kNS][2][kScaleSlot]
  int32_t* smeta = reinterpret_cast<int32_t*>(sscale + (C::kFp8 ? C::kNS * 2 * kScaleSlot : 0));  // [kNS][2]
  uint32_t* smask = reinterpret_cast<uint32_t*>(smeta + 2 * C::kNS);  // gather: [kNS][8]
  uint32_t* shist = smask + (GATHER ? 8 * C::kNS : 0);
  uint64_t* bars = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(shist) + C::kHistBytes);
  // Item it fills stage it % kNS and signals full[it % (2 kNS)]: with two MMA
  // issuers (and two epilogue groups) taking alternate items, successive uses
  // of one stage alternate between them whenever kNS is odd, and a waiter on
  // a shared barrier could then test a phase one ahead of the one completing
  // (the parity would read "done").  Over 2 kNS barriers each barrier's uses
  // are 2 kNS items apart: the same issuer and group wait for every phase.
  uint64_t* full = bars;
  uint64_t* empty = full + 2 * C::kNS;
  uint64_t* qfull = empty + C::kNS;
  uint64_t* qempty = qfull + C::kNQ;
  uint64_t* tfull = qempty + C::kNQ;
  uint64_t* tempty = tfull + C::kAcc;
  uint64_t* done = tempty + C::kAcc;
  uint64_t* ebar = done + 1;  // epilogue warps' rendezvous around histogram flushes
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ebar + 1);
  int* sfound = const_cast<int*>(abort_flag) + 1;                       // 2 ints
  int64_t* sbuf = reinterpret_cast<int64_t*>(sfound + 2 + 1);           // NTH/32 int64 (8-aligned below)
  sbuf = reinterpret_cast<int64_t*>((reinterpret_cast<uintptr_t>(sbuf) + 7) & ~uintptr_t(7));
  // pooled schedule: the ring (kRing segments: barriers, then slots of
  // kSlotInts ints) and the rows' first tiles and visible positions
  uint64_t* rfull = reinterpret_cast<uint64_t*>(sbuf + NTH / 32);
  uint64_t* rempty = rfull + kRing;
  int* rslot = reinterpret_cast<int*>(rempty + kRing);
  int* pool_start = rslot + kRing * kSlotInts;  // [2][kPoolRows]
  const bool pooled = C::kPool && a.pool != nullptr && a.pool_chunk > 0 && a.rows <= kPoolRows;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // a decode step's top-k may be scheduled onto SMs this launch frees (it
  // waits for the scan to complete before reading anything)
  tc::griddep_launch_dependents();
  // The epilogue reads a stage's key rows (paged cache) and scales (FP8); a
  // contiguous bf16 cache needs neither, and its stages free at MMA completion.
  const bool stage_meta = C::kFp8 || a.cache.block_size > 0 || GATHER;
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2 * C::kNS; ++s) {
      // gather: one cp.async completion per producer lane, plus lane 0's masks
      tc::mbar_init(&full[s], GATHER ? 32 + 1 : 1);
    }
    for (int s = 0; s < C::kNS; ++s)
      tc::mbar_init(&empty[s], stage_meta ? 1 + 4 : 1);  // MMA commit (+ 4 epilogue warps done with the stage)
    for (int s = 0; s < C::kNQ; ++s) {
      tc::mbar_init(&qfull[s], 1);
      tc::mbar_init(&qempty[s], 2 + 4 * EG);  // both MMA issuers' commits + every epilogue warp
    }
    for (int s = 0; s < C::kAcc; ++s) {
      tc::mbar_init(&tfull[s], 1);
      tc::mbar_init(&tempty[s], 4);
    }
    tc::mbar_init(done, 2);  // both MMA issuers
    tc::mbar_init(ebar, 4 * EG);
    if (pooled) {
      for (int s = 0; s < kRing; ++s) {
        tc::mbar_init(&rfull[s], 1);            // the producer's publication
        tc::mbar_init(&rempty[s], 3 + 4 * EG);  // both MMA issuers, the query warp, every epilogue warp
      }
    }
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (!GATHER && warp == kWarpProd && lane == 0) {
    tc::prefetch_tmap(&tmap);
    if (C::kFp8) tc::prefetch_tmap(&smap);
  }
  const Plan plan = plan_work<QB, NTH>(a, sbuf, sfound, pooled ? pool_start : nullptr);
  scan_sync<NTH>();
  tc::tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  CacheAddr ad{a.cache.block_table, a.cache.max_blocks, a.cache.block_size, a.cache.n_blocks, a.cache.max_len};
  // Pooled segment k (k = 0, 1, ...) from the ring into a walker and its item
  // count (0: no more); every calling thread reads it, and each consumer
  // releases the slot afterwards (ring_release, once per consumer).
  auto ring_take = [&](int k, Walker<QB>* w, int64_t* n) -> bool {
    const int s = k % kRing;
    if (!tc::mbar_wait(&rfull[s], static_cast<uint32_t>((k / kRing) & 1), abort_flag)) return false;
    const volatile int* sl = rslot + s * kSlotInts;
    Group g;
    g.r0 = sl[0];
    g.nrows = 1;
    g.b = sl[3];
    g.tiles = sl[4];
    g.vis = static_cast<int64_t>(static_cast<uint32_t>(sl[5])) | (static_cast<int64_t>(sl[6]) << 32);
    w->start(g, sl[1]);
    *n = sl[2];
    return true;
  };
  auto ring_release = [&](int k) { tc::mbar_arrive(&rempty[k % kRing]); };

  if (GATHER && warp == kWarpProd) {
    gather_producer<C>(a, plan, ad, stages, smask, full, empty, abort_flag, lane);
  } else if (warp == kWarpProd) {
    // The whole warp looks up the block-table entries of 32 tiles at a time
    // (one tile per lane) and lane 0 issues their TMA loads.  The next batch's
    // entries are loaded before the current batch is issued and only read
    // after it, so their latency hides behind the 32 issues; a single thread
    // doing the lookups serially would wait one load latency per tile.
    // A pooled launch continues past the CTA's static share with chunks of
    // pool_chunk tiles claimed from the pool: the claim for the next chunk is
    // made when the current segment's last batch starts, and the chunk is
    // mapped to its row, published to the other roles and looked up halfway
    // through that batch's issues.
    if (plan.n_items > 0 || pooled) {
      struct Look {
        int64_t p0, vis;  // first position of the tile; visible positions of its group
        int b, r0;
        int32_t blk[2];   // block-table entries of the tile's two boxes (paged cache)
        bool live;
      };
      // lanes [0, left) take the items base, base + 1, ...
      auto look = [&](const Walker<QB>& base, int64_t left) -> Look {
        Look L;
        L.live = lane < left;
        Walker<QB> w = base;
        if (L.live) {
          if (w.j + lane < w.g.tiles) w.j += lane;  // same group: no walk
          else
            for (int i = 0; i < lane; ++i) w.next(a);
        }
        L.p0 = static_cast<int64_t>(w.j) * kTile;
        L.vis = w.g.vis;
        L.b = w.g.b;
        L.r0 = w.g.r0;
        L.blk[0] = L.blk[1] = -1;
        if (L.live && ad.block_size > 0) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int64_t p = L.p0 + h * kBoxRows;
            const int64_t lb = p / ad.block_size;
            if (p < L.vis && lb < ad.max_blocks)
              L.blk[h] = __ldg(ad.block_table + static_cast<int64_t>(L.b) * ad.max_blocks + lb);
          }
        }
        return L;
      };
      // Key rows of the two boxes: >= 0 a row, -3 past the visible range, -2 no such item.
      auto resolve = [&](const Look& L, int64_t* rows) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int64_t p = L.p0 + h * kBoxRows;
          int64_t r = -2;
          if (L.live) {
            if (p >= L.vis) {
              r = -3;
            } else if (ad.block_size == 0) {
              r = static_cast<int64_t>(L.b) * ad.max_len + p;
            } else {
              const int64_t lb = p / ad.block_size;
              const int32_t blk = L.blk[h];
              r = (lb < ad.max_blocks && blk >= 0 && blk < ad.n_blocks)
                      ? static_cast<int64_t>(blk) * ad.block_size + (p - lb * ad.block_size)
                      : -1;
              if (r == -1) record_error(a.status, LSA_ERR_BOUNDS, L.r0, static_cast<int>(p));
            }
          }
          rows[h] = r;
        }
      };
      int claim = 0;  // lane 0: the chunk index returned by the last claim
      int k_pub = 0;  // pooled segments published
      // The claimed chunk as the next segment (0 items: the pool is empty),
      // published to the other roles; false on a timeout.
      auto next_pooled = [&](Walker<QB>* w, int64_t* n) -> bool {
        int r0 = 0, j0 = 0, nn = 0;
        if (lane == 0) {
          const int64_t t0 = plan.pool_lo + static_cast<int64_t>(claim) * a.pool_chunk;
          if (t0 < plan.pool_hi) {
            nn = plan.pool_hi - t0 < a.pool_chunk ? static_cast<int>(plan.pool_hi - t0) : a.pool_chunk;
            // the row holding tile t0: the last row starting at or before it
            int lo = 0, hi = a.rows - 1;
            while (lo < hi) {
              const int mid = (lo + hi + 1) >> 1;
              if (pool_start[mid] <= t0) lo = mid;
              else hi = mid - 1;
            }
            r0 = lo;
            j0 = static_cast<int>(t0 - pool_start[lo]);
          }
        }
        r0 = __shfl_sync(0xffffffffu, r0, 0);
        j0 = __shfl_sync(0xffffffffu, j0, 0);
        nn = __shfl_sync(0xffffffffu, nn, 0);
        Group g;
        g.r0 = r0;
        g.nrows = 1;
        g.b = seq_of(a, r0);
        g.vis = pool_start[kPoolRows + r0];
        g.tiles = static_cast<int>((g.vis + kTile - 1) / kTile);
        bool ok = true;
        if (lane == 0) {
          const int s = k_pub % kRing;
          ok = tc::mbar_wait(&rempty[s], static_cast<uint32_t>(((k_pub / kRing) & 1) ^ 1), abort_flag);
          if (ok) {
            int* sl = rslot + s * kSlotInts;
            sl[0] = g.r0;
            sl[1] = j0;
            sl[2] = nn;
            sl[3] = g.b;
            sl[4] = g.tiles;
            sl[5] = static_cast<int>(static_cast<uint32_t>(g.vis));
            sl[6] = static_cast<int>(g.vis >> 32);
            tc::mbar_arrive(&rfull[s]);  // release: the slot is visible to the consumers' acquire
          } else {
            record_error(a.status, LSA_ERR_TIMEOUT, 0, 10);
            *abort_flag = 1;
          }
        }
        ++k_pub;
        w->start(g, j0);
        *n = nn;
        return __shfl_sync(0xffffffffu, ok, 0);
      };
      // decode streams each key once per step: evict it first; the causal
      // prefill reads every key once per group of query rows: keep it
      const uint64_t l2_policy = a.row_pos ? tc::l2_evict_last_policy() : tc::l2_evict_first_policy();
      int64_t it = 0;
      bool failed = false;
      // Issues item i of the batch whose key rows the lanes hold; false on a timeout.
      auto issue = [&](const int64_t* cur_rows, int i) -> bool {
        const int64_t rows[2] = {__shfl_sync(0xffffffffu, cur_rows[0], i), __shfl_sync(0xffffffffu, cur_rows[1], i)};
        bool bad = false;
        if (lane == 0) {
          const int s = static_cast<int>(it % C::kNS);
          const uint32_t ph = static_cast<uint32_t>((it / C::kNS) & 1);
          uint64_t* fb = &full[it % (2 * C::kNS)];
          if (!tc::mbar_wait(&empty[s], ph ^ 1, abort_flag)) {
            record_error(a.status, LSA_ERR_TIMEOUT, 0, 1);
            *abort_flag = 1;
            bad = true;
          } else {
            uint32_t bytes = 0;
            for (int h = 0; h < 2; ++h)
              if (rows[h] >= 0) bytes += C::kKBlocks * C::kBoxBytes + (C::kFp8 ? kScaleBox * 4 : 0);
            smeta[2 * s] = static_cast<int32_t>(rows[0]);  // published to the epilogue by the full barrier
            smeta[2 * s + 1] = static_cast<int32_t>(rows[1]);
            tc::mbar_arrive_expect_tx(fb, bytes);
            uint8_t* st = stages + s * C::kTileBytes;
            for (int h = 0; h < 2; ++h) {
              if (rows[h] < 0) continue;
              for (int kb = 0; kb < C::kKBlocks; ++kb)
                tc::tma_load_2d_hint(st + kb * C::kKBlockBytes + h * C::kBoxBytes, &tmap, kb * kBoxX,
                                     static_cast<int32_t>(rows[h]), fb, l2_policy);
              // the box's 64 scales, from the 16-byte aligned row at or below its first
              if (C::kFp8)
                tc::tma_load_1d(sscale + (2 * s + h) * kScaleSlot, &smap, static_cast<int32_t>(rows[h] & ~int64_t(3)),
                                fb);
            }
            ++it;
          }
        }
        return !__shfl_sync(0xffffffffu, bad, 0);
      };
      Walker<QB> Wb;
      int64_t left = plan.n_items;  // items of the current segment from Wb on
      if (left > 0) {
        Wb.start(a, plan.r_first, plan.j_first);
      } else {  // no static share: the first segment comes from the pool
        if (lane == 0) claim = atomicAdd(a.pool, 1);
        failed = !next_pooled(&Wb, &left);
      }
      Look cur = look(Wb, left);
      while (left > 0 && !failed) {
        int64_t cur_rows[2];
        resolve(cur, cur_rows);
        const int nb = static_cast<int>(left < 32 ? left : 32);
        // The next batch: the rest of this segment, else the next pooled
        // segment (claimed now, mapped after the first half of the issues).
        const bool to_pool = pooled && nb == left;
        if (to_pool && lane == 0) claim = atomicAdd(a.pool, 1);
        const int h = to_pool ? (nb + 1) / 2 : 0;
        for (int i = 0; i < h && !failed; ++i) failed = !issue(cur_rows, i);
        Walker<QB> Wn = Wb;
        int64_t nleft = left - nb;
        if (failed) break;
        if (nleft > 0) {
          if (Wn.j + 32 < Wn.g.tiles) Wn.j += 32;
          else
            for (int i = 0; i < 32; ++i) Wn.next(a);
        } else if (to_pool) {
          if (!next_pooled(&Wn, &nleft)) break;
        }
        const Look nxt = look(Wn, nleft);  // loads stay in flight during the issues below
        for (int i = h; i < nb && !failed; ++i) failed = !issue(cur_rows, i);
        Wb = Wn;
        left = nleft;
        cur = nxt;
      }
      // drain: the last load of every stage must land before the CTA exits
      if (lane == 0) {
        const int64_t n_issued = it;
        for (int64_t i = n_issued > C::kNS ? n_issued - C::kNS : 0; i < n_issued; ++i)
          tc::mbar_wait(&full[i % (2 * C::kNS)], static_cast<uint32_t>((i / (2 * C::kNS)) & 1), nullptr);
      }
    }
  } else if (warp == kWarpMma || warp == warp_mma2<EG>()) {
    // issuer `who` takes the tiles it with it % 2 == who, into accumulator it % kAcc
    const int who = warp == kWarpMma ? 0 : 1;
    if (lane == 0 && (plan.n_items > 0 || pooled)) {
      Walker<QB> W;
      int64_t n = plan.n_items;  // items of the current segment
      if (n > 0) W.start(a, plan.r_first, plan.j_first);
      int gi = -1;
      int qi = 0;
      // An issuer shares its SM sub-partition with epilogue warps, so its
      // per-tile work is kept small: the stage and its phase advance
      // incrementally (no 64-bit division per tile), and a tile's descriptors
      // are the first stage's and query buffer's plus constant offsets in the
      // start-address field (shared-memory addresses stay below 256 KB: adding
      // never carries out of that 14-bit field).
      // the item's stage, and the passes over the stages so far (mod 4): its
      // full barrier is s + kNS (sweep & 1), that barrier's phase sweep >> 1
      int s = 0;
      uint32_t sweep = 0;
      const uint64_t a_desc0 = tc::desc_sw128(tc::smem_u32(stages));
      const uint64_t b_desc0 = tc::desc_sw128(tc::smem_u32(qbufs));
      int64_t it = 0;  // items of every segment so far
      bool fail = false;
      for (int k = 0;; ++k) {
        for (int64_t i = 0; i < n; ++i, ++it) {
          if (i == 0 || W.j == 0) {
            ++gi;
            qi = gi % C::kNQ;
            if (!tc::mbar_wait(&qfull[qi], static_cast<uint32_t>((gi / C::kNQ) & 1), abort_flag)) {
              fail = true;
              break;
            }
          }
          if (static_cast<int>(it & 1) == who) {
            if (!tc::mbar_wait(&full[s + C::kNS * (sweep & 1u)], sweep >> 1, abort_flag)) {
              fail = true;
              break;
            }
            // gathered rows were written by cp.async (generic proxy); the MMA reads them through the async proxy
            if (GATHER) tc::fence_proxy_async_smem();
            const int acc = static_cast<int>(it % C::kAcc);
            if (!tc::mbar_wait(&tempty[acc], static_cast<uint32_t>(((it / C::kAcc) & 1) ^ 1), abort_flag)) {
              fail = true;
              break;
            }
            tc::tc_fence_after();
            const uint32_t d = tmem_base + acc * C::kAccCols;
            const uint64_t ad0 = a_desc0 + static_cast<uint64_t>((s * C::kTileBytes) >> 4);
            const uint64_t bd0 = b_desc0 + static_cast<uint64_t>((qi * C::kQBytes) >> 4);
            if (C::kCat) {
              // D = K q_hi + K q_lo: the query operand's rows 64-127 start 8 KB in
#pragma unroll
              for (int part = 0; part < 2; ++part) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t ad_ = ad0 + static_cast<uint64_t>((kk * 32) >> 4);
                  const uint64_t bd_ = bd0 + static_cast<uint64_t>((part * kHeads * 128 + kk * 32) >> 4);
                  tc::mma_f8(d, ad_, bd_, C::kIdesc, (part | kk) != 0);
                }
              }
            } else {
#pragma unroll
              for (int kb = 0; kb < C::kKBlocks; ++kb) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                  const uint64_t ad_ = ad0 + static_cast<uint64_t>((kb * C::kKBlockBytes + kk * 32) >> 4);
                  const uint64_t bd_ = bd0 + static_cast<uint64_t>((kb * C::kQKBlockBytes + kk * 32) >> 4);
                  if (C::kFp8) tc::mma_f8(d, ad_, bd_, C::kIdesc, (kb | kk) != 0);
                  else tc::mma_f16(d, ad_, bd_, C::kIdesc, (kb | kk) != 0);
                }
              }
            }
            tc::mma_commit(&empty[s]);
            tc::mma_commit(&tfull[acc]);
          }
          if (++s == C::kNS) {
            s = 0;
            sweep = (sweep + 1u) & 3u;
          }
          // both issuers release the group's query buffer after its last tile
          // of the segment (a commit covers every MMA its thread issued before it)
          if (i + 1 == n || W.j + 1 >= W.g.tiles) tc::mma_commit(&qempty[qi]);
          if (i + 1 < n) W.next(a);
        }
        if (fail || !pooled) break;
        if (!ring_take(k, &W, &n)) {
          fail = true;
          break;
        }
        ring_release(k);
        if (n == 0) break;
      }
      if (fail) {
        record_error(a.status, LSA_ERR_TIMEOUT, 0, 2);
        *abort_flag = 1;
      }
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, nullptr);  // both issuers' MMAs complete
      // The releases of the last stages and query buffer arrive asynchronously
      // too; they must land before the barriers are invalidated.
      if (who == 0 && !*abort_flag) {
        for (int64_t i = it > C::kNS ? it - C::kNS : 0; i < it; ++i)
          tc::mbar_wait(&empty[i % C::kNS], static_cast<uint32_t>((i / C::kNS) & 1), abort_flag);
        if (gi >= 0) tc::mbar_wait(&qempty[gi % C::kNQ], static_cast<uint32_t>((gi / C::kNQ) & 1), abort_flag);
      }
    }
  } else if (warp == kWarpQ) {
    if (plan.n_items > 0 || pooled) {
      Walker<QB> W;
      int64_t n = plan.n_items;  // items of the current segment
      if (n > 0) W.start(a, plan.r_first, plan.j_first);
      int gi = -1;
      bool fail = false;
      for (int k = 0;; ++k) {
        for (int64_t i = 0; i < n; ++i) {
          if (i == 0 || W.j == 0) {
            ++gi;
            const int qi = gi % C::kNQ;
            if (!tc::mbar_wait(&qempty[qi], static_cast<uint32_t>(((gi / C::kNQ) & 1) ^ 1), abort_flag)) {
              if (lane == 0) {
                record_error(a.status, LSA_ERR_TIMEOUT, 0, 3);
                *abort_flag = 1;
              }
              fail = true;
              break;
            }
            uint8_t* qb = qbufs + qi * C::kQBytes;
            float* wb = wbufs + qi * (C::kWBytes / 4);
            if (C::kFp8) stage_query_fp8<QB>(a, W.g, qb, wb, qraw, lane);
            else stage_query_bf16<QB>(a, W.g, qb, wb, lane);
            tc::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&qfull[qi]);
          }
          if (i + 1 < n) W.next(a);
        }
        if (fail || !pooled) break;
        if (!ring_take(k, &W, &n)) {
          if (lane == 0) {
            record_error(a.status, LSA_ERR_TIMEOUT, 0, 11);
            *abort_flag = 1;
          }
          break;
        }
        __syncwarp();
        if (lane == 0) ring_release(k);
        if (n == 0) break;
      }
    }
  } else if (warp < kWarpEpi + 4 * EG) {
    // epilogue: warp % 4 selects the TMEM lane quarter = token rows of the
    // tile; group eg (warps 3 + 4 eg ..) takes the tiles it with it % EG == eg
    const int quarter = warp & 3;
    const int eg = (warp - kWarpEpi) / 4;
    const int t = quarter * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    // Decode with a histogram target: the epilogue also counts each score's
    // top-k digit (key bits [31:20]) in shared memory and adds the counts of a
    // row to hist12 when the CTA leaves that row, so the top-k skips one pass.
    const bool use_hist = QB == 1 && a.hist12 != nullptr;
    const int et = threadIdx.x - kWarpEpi * 32;  // 0 .. 128 EG - 1
    int ephase = 0;
    auto epi_sync = [&]() -> bool {
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(ebar);
      const bool ok = tc::mbar_wait(ebar, static_cast<uint32_t>(ephase & 1), abort_flag);
      ++ephase;
      return ok;
    };
    auto flush_hist = [&](int row) -> bool {
      if (!epi_sync()) return false;
      uint32_t* dst = a.hist12 + static_cast<int64_t>(row) * kTopkBins1;
      for (int i = et; i < kTopkBins1; i += 128 * EG) {
        const uint32_t v = shist[i];
        if (v) {
          atomicAdd(dst + i, v);
          shist[i] = 0;
        }
      }
      return epi_sync();
    };
    if (use_hist)
      for (int i = et; i < kTopkBins1; i += 128 * EG) shist[i] = 0;
    // Tails first (the epilogue warps wait for their first accumulator
    // anyway): positions past each row's group tiles are -inf, the whole row
    // NaN for an invalid row.  No tile writes there, so the order is free.
    for (int r = blockIdx.x; r < a.rows; r += gridDim.x) {
      int r0 = r;
      while (!is_leader<QB>(a, r0)) --r0;
      const Group g = group_at<QB>(a, r0);
      int b;
      row_visible(a, r, &b);
      const bool ok = b >= 0 && b < a.cache.batch;
      if (ok && et == 0) {
        const int L = __ldg(a.cache.seq_lens + b);
        if (L < 0 || L > a.cache.max_len) record_error(a.status, LSA_ERR_BOUNDS, r, L);
      } else if (!ok && et == 0) {
        record_error(a.status, LSA_ERR_BOUNDS, r, b);
      }
      const float val = ok ? -INFINITY : NAN;
      int64_t start = ok ? static_cast<int64_t>(g.tiles) * kTile : 0;
      start = start < a.ld ? start : a.ld;
      float* row = a.scores + static_cast<int64_t>(r) * a.ld;
      const int64_t mis = (reinterpret_cast<uintptr_t>(row + start) >> 2) & 3;  // floats to 16-byte alignment
      int64_t head = start + ((4 - mis) & 3);
      head = head < a.ld ? head : a.ld;
      for (int64_t p = start + et; p < head; p += 128 * EG) row[p] = val;
      const int64_t nvec = (a.ld - head) >> 2;
      float4* v4 = reinterpret_cast<float4*>(row + head);
      for (int64_t i = et; i < nvec; i += 128 * EG) v4[i] = make_float4(val, val, val, val);
      for (int64_t p = head + nvec * 4 + et; p < a.ld; p += 128 * EG) row[p] = val;
    }
    if (plan.n_items > 0 || pooled) {
      Walker<QB> W;
      int64_t n = plan.n_items;  // items of the current segment
      if (n > 0) W.start(a, plan.r_first, plan.j_first);
      int gi = -1, qi = 0;
      int hist_row = -1;
      int32_t vis_r[QB];  // visible positions of the group's rows (below 2^31)
      int stg = 0;          // stage of item it
      uint32_t sweep = 0;   // passes over the stages (mod 4): full barrier and phase, as the issuers
      int64_t it = 0;     // items of every segment so far
      bool fail = false;
      for (int k = 0;; ++k) {
        // `left` counts the segment's items down (fewer live 64-bit registers
        // in the epilogue than an index and a bound)
        bool seg_first = true;
        for (int64_t left = n; left > 0; --left, ++it) {
          if (seg_first || W.j == 0) {
            seg_first = false;
            ++gi;
            qi = gi % C::kNQ;
            // a new row: the counts of the one before go to its histogram
            if (use_hist && hist_row >= 0 && hist_row != W.g.r0 && !flush_hist(hist_row)) {
              if (lane == 0) {
                record_error(a.status, LSA_ERR_TIMEOUT, 0, 6);
                *abort_flag = 1;
              }
              hist_row = -1;
              fail = true;
              break;
            }
            hist_row = W.g.r0;
            if (!tc::mbar_wait(&qfull[qi], static_cast<uint32_t>((gi / C::kNQ) & 1), abort_flag)) {
              if (lane == 0) {
                record_error(a.status, LSA_ERR_TIMEOUT, 0, 4);
                *abort_flag = 1;
              }
              hist_row = -1;
              fail = true;
              break;
            }
            if (QB == 1) {
              vis_r[0] = static_cast<int32_t>(W.g.vis);  // the group's one row
            } else {
#pragma unroll
              for (int qq = 0; qq < QB; ++qq) {
                int bb;
                vis_r[qq] = qq < W.g.nrows ? static_cast<int32_t>(row_visible(a, W.g.r0 + qq, &bb)) : 0;
              }
            }
          }
          // the other group's tiles are only walked past (both groups release
          // every query buffer: the weights are read by either)
          const bool mine = EG == 1 || static_cast<int>(it % EG) == eg;
          if (mine) {
            const int acc = static_cast<int>(it % C::kAcc);
            if (!tc::mbar_wait(&tfull[acc], static_cast<uint32_t>((it / C::kAcc) & 1), abort_flag)) {
              if (lane == 0) {
                record_error(a.status, LSA_ERR_TIMEOUT, 0, 5);
                *abort_flag = 1;
              }
              hist_row = -1;
              fail = true;
              break;
            }
            tc::tc_fence_after();
            // The tile's key rows (and FP8 scales) come from the producer through
            // the stage; the stage is released once all four warps have read them.
            int32_t mrow = 0;  // contiguous bf16: every visible position has a key row
            float kscale = 1.f;
            if (stage_meta) {
              if (!tc::mbar_wait(&full[stg + C::kNS * (sweep & 1u)], sweep >> 1, abort_flag)) {
                if (lane == 0) {
                  record_error(a.status, LSA_ERR_TIMEOUT, 0, 8);
                  *abort_flag = 1;
                }
                hist_row = -1;
                fail = true;
                break;
              }
              if (GATHER) {
                // row t has a key (0), is a padding entry (-3: -inf) or an out-of-range one (-1: NaN)
                const uint32_t* mk = smask + 8 * stg;
                mrow = ((mk[t >> 5] >> (t & 31)) & 1u) ? 0 : (((mk[4 + (t >> 5)] >> (t & 31)) & 1u) ? -1 : -3);
              } else {
                const int box = 2 * stg + (t >> 6);
                mrow = smeta[box];
                if (C::kFp8 && mrow >= 0) kscale = sscale[box * kScaleSlot + (mrow & 3) + (t & 63)];
              }
              __syncwarp();
              if (lane == 0) tc::mbar_arrive(&empty[stg]);
            }
            const int64_t p = static_cast<int64_t>(W.j) * kTile + t;
            const int64_t prow = mrow >= 0 ? static_cast<int64_t>(mrow) + (t & 63) : (GATHER && mrow == -3 ? -3 : -1);
            const float* wb = wbufs + qi * (C::kWBytes / 4);
            float sc[QB];
#pragma unroll
            for (int qq = 0; qq < QB; ++qq) {
              float s = 0.f;
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                float v[32];
                const uint32_t col =
                    acc * C::kAccCols + (C::kFp8 && !C::kCat ? qq * 2 * kHeads : qq * kHeads) + c * 32;
                tc::tmem_ld32(tmem_base + lane_base + col, v);
                const float4* w4 = reinterpret_cast<const float4*>(wb + qq * kHeads + c * 32);
                if (C::kFp8 && !C::kCat) {
                  float u[32];
                  tc::tmem_ld32(tmem_base + lane_base + col + kHeads, u);
                  tc::tmem_wait_ld();
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const float4 w = w4[i];
                    s = fmaf(w.x, fmaxf(v[4 * i] + u[4 * i], 0.f), s);
                    s = fmaf(w.y, fmaxf(v[4 * i + 1] + u[4 * i + 1], 0.f), s);
                    s = fmaf(w.z, fmaxf(v[4 * i + 2] + u[4 * i + 2], 0.f), s);
                    s = fmaf(w.w, fmaxf(v[4 * i + 3] + u[4 * i + 3], 0.f), s);
                  }
                } else {
                  tc::tmem_wait_ld();
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    const float4 w = w4[i];
                    s = fmaf(w.x, fmaxf(v[4 * i], 0.f), s);
                    s = fmaf(w.y, fmaxf(v[4 * i + 1], 0.f), s);
                    s = fmaf(w.z, fmaxf(v[4 * i + 2], 0.f), s);
                    s = fmaf(w.w, fmaxf(v[4 * i + 3], 0.f), s);
                  }
                }
              }
              sc[qq] = s * kscale;
            }
            tc::tc_fence_before();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&tempty[acc]);
            if (use_hist && p < vis_r[0] && prow >= 0) {
              const uint32_t key = order_key(sc[0]);
              if (key) atomicAdd(&shist[key >> 20], 1u);
            }
#pragma unroll
            for (int qq = 0; qq < QB; ++qq) {
              if (qq < W.g.nrows && p < a.ld) {
                float o = -INFINITY;
                if (p < vis_r[qq]) o = prow >= 0 ? sc[qq] : (prow == -3 ? -INFINITY : NAN);
                a.scores[static_cast<int64_t>(W.g.r0 + qq) * a.ld + p] = o;
              }
            }
          }
          const bool last = left == 1 || (W.j + 1 >= W.g.tiles);
          if (last) {
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&qempty[qi]);
          }
          if (++stg == C::kNS) {
            stg = 0;
            sweep = (sweep + 1u) & 3u;
          }
          if (left > 1) W.next(a);
        }
        if (fail || !pooled) break;
        if (!ring_take(k, &W, &n)) {
          if (lane == 0) {
            record_error(a.status, LSA_ERR_TIMEOUT, 0, 12);
            *abort_flag = 1;
          }
          hist_row = -1;
          break;
        }
        __syncwarp();
        if (lane == 0) ring_release(k);
        if (n == 0) break;
      }
      if (use_hist && hist_row >= 0 && !flush_hist(hist_row) && lane == 0) {
        record_error(a.status, LSA_ERR_TIMEOUT, 0, 7);
        *abort_flag = 1;
      }
    }
  }
  tc::tc_fence_before();
  scan_sync<NTH>();
  if (threadIdx.x == 0) {
    for (uint64_t* b = bars; b <= ebar; ++b) tc::mbar_inval(b);
    if (pooled)
      for (uint64_t* b = rfull; b < rempty + kRing; ++b) tc::mbar_inval(b);
  }
  scan_sync<NTH>();
  if (a.done_ctr) {
    // decode step: the top-k starts on this count instead of the grid's
    // completion; the barrier orders every thread's score stores and histogram
    // adds before thread 0's release
    scan_sync<NTH>();
    if (threadIdx.x == 0) tc::red_release_gpu_add(a.done_ctr, 1u);
  }
}

}  // namespace scan
}  // namespace lsa
