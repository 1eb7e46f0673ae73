#pragma once
// Sparse MQA decode on the sm_100a tensor cores (tcgen05 + TMEM), gathering
// the selected KV rows through the block table.
//
// The layer attends only the k tokens the lightning indexer kept (MLI abstract,
// sentence 2): o[h] = softmax_j(scale * q[h] . KV[idx_j]) . KV[idx_j][:512]
// over 128 query heads sharing 576-wide bf16 KV rows (value = first 512
// columns), plus lse[h].  Sparse attention reads only the kept rows (LeanSparse
// episode page: it reduces reads, not storage).
//
// Work: one CTA per (query row, half of the heads, split of the index list).
// 64 heads make the MMA's M side (M = 64), so the fp32 output accumulator
// O[64 x 512] takes half of the TMEM lanes: dims 0-255 at lane offset 0 and
// dims 256-511 at lane offset 16, columns 0-255; the two score buffers
// S[64 x 64] sit at lane offset 0, columns 256-383.  Each softmax warp then
// holds, for its 16 heads, the scores in lanes 0-15 and both output halves in
// lanes 0-31, so a rescale touches only output columns.
//   warps 0-3  producer: cp.async gathers of 64 selected rows per chunk into the
//              128-byte-swizzled operand layout (two chunk buffers); the rows of
//              chunk j+2 are looked up and prefetched into L2 while chunk j is
//              gathered, so the gathers read L2, not HBM
//   warp 4     MMA issuer: S = Q K^T (36 x M64N64K16), O += P V (8 x M64N256K16),
//              V read MN-major from the same tile as K
//   warps 5-8  online softmax (base 2, lazy rescale when the max grows by > 8),
//              P[64 heads x 64 rows] written over the chunk's rope block (dims
//              512-575, dead once S is computed), so P is double-buffered with
//              the chunks and the softmax of chunk j+1 overlaps P V of chunk j
// (Below N = 64 an MMA costs as much as at N = 64 on this part, so 64-row
// chunks halve the score MMAs per row compared with 32-row chunks.)
// With several splits per row, each CTA writes a normalised partial and its
// lse; the last CTA of a (row, half) to finish merges them with all of its
// threads (global counter, no waiting), so no separate merge launch is needed.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"

namespace lsa {
namespace attn {

constexpr int kHeadsAll = 128;
constexpr int kHeadsCta = 64;
constexpr int kD = 576;
constexpr int kDv = 512;
constexpr int kChunk = 64;                 // KV rows per chunk
constexpr int kNBuf = 2;                   // chunk buffers
constexpr int kBoxes = kD / 64;            // 9 column blocks of 64 dims
constexpr int kBoxBytes = kChunk * 128;    // 64 rows x 128 B
constexpr int kKvBytes = kBoxes * kBoxBytes;          // 73728
constexpr int kQBlock = kHeadsCta * 128;              // 8192
constexpr int kQBytes = kBoxes * kQBlock;             // 73728
constexpr int kRopeBox = kBoxes - 1;                  // column block of dims 512-575; holds P after S
constexpr int kThreads = 288;
constexpr int kProdThreads = 128;
constexpr int kWarpMma = 4;                // warps 5-8: softmax
constexpr int kSmemBytes = kQBytes + kNBuf * kKvBytes + 1024 /*barriers*/ + 1024 /*align*/;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 256;            // score buffers start column
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.f;        // lazy rescale threshold (factor 256)

constexpr uint32_t kIdescQK = tc::idesc(tc::kFmtBF16, tc::kFmtBF16, 64, kChunk);
constexpr uint32_t kIdescPV = tc::idesc(tc::kFmtBF16, tc::kFmtBF16, 64, 256) | (1u << 16);  // B MN-major

static_assert(kSmemBytes <= 232448, "shared memory");

struct TcAttnParams {
  AttnArgs a;
  int nsplit;
  int split_len;   // multiple of kChunk
  float* part_o;   // [rows][nsplit][128][512]
  float* part_lse; // [rows][nsplit][128]
  int* counters;   // [rows][2], zeroed before the launch
};

// MN-major operand in the 128-byte swizzle layout: 64-element MN blocks `lbo`
// bytes apart, 8-row K groups 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128_mn(uint32_t addr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(tc::smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}

// 2^x on the special-function unit (ex2.approx.ftz); 2^-inf = +0.
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

struct RowCtx {
  int b;
  int64_t L;
  bool ok;
};

__device__ __forceinline__ RowCtx row_ctx(const AttnArgs& a, int r) {
  RowCtx c;
  c.b = a.row_seq ? __ldg(a.row_seq + r) : r;
  c.ok = c.b >= 0 && c.b < a.cache.batch;
  c.L = c.ok ? __ldg(a.cache.seq_lens + c.b) : 0;
  if (c.L < 0) c.L = 0;
  if (c.L > a.cache.max_len) c.L = a.cache.max_len;
  return c;
}

// Stored rows of list entries j[0..N) of row r (-1: padding, out of range or
// bad block).  All index loads are issued before the block-table loads.
template <int N>
__device__ __forceinline__ void entry_rows(const AttnArgs& a, const CacheAddr& ad, const RowCtx& rc, int r,
                                           const int (&j)[N], int j1, bool report, int64_t (&out)[N]) {
  int32_t pos[N];
#pragma unroll
  for (int m = 0; m < N; ++m)
    // L2-coherent load: in the fused step the selection is written earlier in the same launch
    pos[m] = (j[m] < j1 && rc.ok) ? __ldcg(a.idx + static_cast<int64_t>(r) * a.k + j[m]) : -1;
  if (ad.block_size == 0) {
#pragma unroll
    for (int m = 0; m < N; ++m) out[m] = (pos[m] >= 0 && pos[m] < rc.L) ? static_cast<int64_t>(rc.b) * ad.max_len + pos[m] : -1;
  } else {
    int32_t blk[N];
#pragma unroll
    for (int m = 0; m < N; ++m) {
      const int64_t lb = pos[m] / ad.block_size;
      blk[m] = (pos[m] >= 0 && pos[m] < rc.L && lb < ad.max_blocks)
                   ? __ldg(ad.block_table + static_cast<int64_t>(rc.b) * ad.max_blocks + lb) : -1;
    }
#pragma unroll
    for (int m = 0; m < N; ++m)
      out[m] = (blk[m] >= 0 && blk[m] < ad.n_blocks)
                   ? static_cast<int64_t>(blk[m]) * ad.block_size + (pos[m] % ad.block_size) : -1;
  }
  if (report) {
#pragma unroll
    for (int m = 0; m < N; ++m)
      if (pos[m] >= 0 && out[m] < 0) record_error(a.status, LSA_ERR_BOUNDS, r, pos[m]);
  }
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* o, const float (&v)[32], float inv) {
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const __nv_bfloat162 pb = __floats2bfloat162_rn(v[u * 8 + 2 * e] * inv, v[u * 8 + 2 * e + 1] * inv);
      w[e] = *reinterpret_cast<const uint32_t*>(&pb);
    }
    *reinterpret_cast<uint4*>(o + u * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// One CTA of the sparse attention: 64 heads (`half`) of query row r over the
// split-th range of its selection.  `tmem_slot` holds (or, once the first block
// barrier has passed, will hold) the base of kTmemCols allocated TMEM columns.
// Every mbarrier it used is invalidated before it returns, so the caller may
// reuse the shared memory.
__device__ __forceinline__ void attn_cta(const TcAttnParams& P, uint8_t* smem_raw, int split, int half, int r,
                                         const volatile uint32_t* tmem_slot) {
  const AttnArgs& a = P.a;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* qs = smem;
  uint8_t* kvs = qs + kQBytes;         // kNBuf chunk buffers
  uint64_t* bars = reinterpret_cast<uint64_t*>(kvs + kNBuf * kKvBytes);
  uint64_t* qfull = bars;
  uint64_t* kvfull = bars + 1;            // [kNBuf]
  uint64_t* kvempty = kvfull + kNBuf;     // [kNBuf]
  uint64_t* sfull = kvempty + kNBuf;      // [2]
  uint64_t* sempty = sfull + 2;           // [2]
  uint64_t* pfull = sempty + 2;
  uint64_t* pvdone = pfull + 1;
  uint64_t* done = pvdone + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(done + 1);
  int* last_flag = const_cast<int*>(abort_flag) + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = split * P.split_len;
  const int j1 = min(a.k, j0 + P.split_len);
  const int nch = j1 > j0 ? (j1 - j0 + kChunk - 1) / kChunk : 0;

  if (threadIdx.x == 0) {
    tc::mbar_init(qfull, kProdThreads);
    for (int i = 0; i < kNBuf; ++i) {
      tc::mbar_init(&kvfull[i], kProdThreads);
      tc::mbar_init(&kvempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(&sfull[i], 1);
      tc::mbar_init(&sempty[i], 4);
    }
    tc::mbar_init(pfull, 4);
    tc::mbar_init(pvdone, 1);
    tc::mbar_init(done, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const RowCtx rc = row_ctx(a, r);
  CacheAddr ad{a.cache.block_table, a.cache.max_blocks, a.cache.block_size, a.cache.n_blocks, a.cache.max_len};
  if (!rc.ok && threadIdx.x == 0 && split == 0 && half == 0) record_error(a.status, LSA_ERR_BOUNDS, r, rc.b);

  if (warp < 4) {
    // ---------------------------------------------------------------- producer
    const int t = threadIdx.x;
    const int sub = t & 7;         // 16-byte column chunk within each 128-byte block
    const int rbase = t >> 3;      // 0..15
    const bool report = sub == 0 && half == 0;
    // rows of this thread (4 per chunk) for chunks j, j+1 and j+2
    int64_t rc_[4], rn_[4], rn2_[4];
    auto lookup = [&](int jj, int64_t (&dst)[4]) {
      int jl[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) jl[m] = jj < nch ? j0 + jj * kChunk + rbase + 16 * m : j1;
      entry_rows<4>(a, ad, rc, r, jl, j1, report, dst);
    };
    auto prefetch_l2 = [&](const int64_t (&rows)[4]) {
      if (sub != 0) return;
#pragma unroll
      for (int m = 0; m < 4; ++m)
        if (rows[m] >= 0)
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                           reinterpret_cast<const uint8_t*>(a.cache.kv) + rows[m] * (kD * 2)),
                       "r"(kD * 2)
                       : "memory");
    };
    // the first three chunks' lookups go out before the query copy, so their
    // latency overlaps it
    lookup(0, rc_);
    lookup(1, rn_);
    lookup(2, rn2_);
    const uint8_t* qsrc = reinterpret_cast<const uint8_t*>(a.q) +
                          (static_cast<int64_t>(r) * kHeadsAll + half * kHeadsCta) * kD * 2;
    const uint32_t qs_u = tc::smem_u32(qs);
    for (int m = 0; m < 4; ++m) {
      const int i = rbase + 16 * m;
      const uint8_t* src = qsrc + static_cast<int64_t>(i) * kD * 2;
      for (int d = 0; d < kBoxes; ++d)
        cp_async16(qs_u + d * kQBlock + tc::sw128_offset(i, sub), src + d * 128 + sub * 16);
    }
    cp_async_arrive_noinc(qfull);
    prefetch_l2(rc_);
    prefetch_l2(rn_);
    for (int j = 0; j < nch; ++j) {
      const int b = j % kNBuf;
      prefetch_l2(rn2_);  // chunk j+2 (looked up during the previous iteration)
      if (!tc::mbar_wait(&kvempty[b], ((j / kNBuf) & 1) ^ 1, abort_flag)) {
        if (t == 0) {
          record_error(a.status, LSA_ERR_TIMEOUT, r, 10);
          *abort_flag = 1;
        }
        break;
      }
      uint8_t* kvb = kvs + b * kKvBytes;
      const uint32_t kv_u = tc::smem_u32(kvb);
      bool zeroed = false;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = rbase + 16 * m;
        if (rc_[m] >= 0) {
          const uint8_t* src = reinterpret_cast<const uint8_t*>(a.cache.kv) + rc_[m] * (kD * 2);
#pragma unroll
          for (int d = 0; d < kBoxes; ++d)
            cp_async16(kv_u + d * kBoxBytes + tc::sw128_offset(i, sub), src + d * 128 + sub * 16);
        } else {
#pragma unroll
          for (int d = 0; d < kBoxes; ++d)
            *reinterpret_cast<uint4*>(kvb + d * kBoxBytes + tc::sw128_offset(i, sub)) = make_uint4(0, 0, 0, 0);
          zeroed = true;
        }
      }
      if (zeroed) tc::fence_proxy_async_smem();
      cp_async_arrive_noinc(&kvfull[b]);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        rc_[m] = rn_[m];
        rn_[m] = rn2_[m];
      }
      lookup(j + 3, rn2_);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0 && nch > 0) {
      const uint32_t q_u = tc::smem_u32(qs);
      bool ok = tc::mbar_wait(qfull, 0, abort_flag);
      tc::fence_proxy_async_smem();
      auto issue_pv = [&](int i) -> bool {
        if (!tc::mbar_wait(pfull, i & 1, abort_flag)) return false;
        tc::tc_fence_after();
        const uint32_t kv_u = tc::smem_u32(kvs + (i % kNBuf) * kKvBytes);
        const uint32_t p_u = kv_u + kRopeBox * kBoxBytes;  // P(i) sits in chunk i's rope block
        const uint64_t pa0 = tc::desc_sw128(p_u), vb0 = desc_sw128_mn(kv_u, kBoxBytes);
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const uint32_t d = tmem + (static_cast<uint32_t>(16 * c) << 16);  // dims 256c.. at lane offset 16c
#pragma unroll
          for (int kk = 0; kk < kChunk / 16; ++kk)
            tc::mma_f16(d, pa0 + static_cast<uint64_t>((kk * 32) >> 4),
                        vb0 + static_cast<uint64_t>(((4 * c) * kBoxBytes + kk * 2048) >> 4), kIdescPV,
                        (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc::mma_commit(pvdone);
        tc::mma_commit(&kvempty[i % kNBuf]);
        return true;
      };
      for (int j = 0; ok && j < nch; ++j) {
        const int b = j % kNBuf, sb = j & 1;
        if (!tc::mbar_wait(&kvfull[b], (j / kNBuf) & 1, abort_flag)) { ok = false; break; }
        tc::fence_proxy_async_smem();
        if (!tc::mbar_wait(&sempty[sb], ((j >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
        tc::tc_fence_after();
        const uint32_t kv_u = tc::smem_u32(kvs + b * kKvBytes);
        const uint32_t d = tmem + kColS + sb * kChunk;
        // descriptors of the 36 K-steps differ only in the start-address field
        // (addresses stay below 256 KB, so the 14-bit field never carries)
        const uint64_t a0 = tc::desc_sw128(q_u), b0 = tc::desc_sw128(kv_u);
#pragma unroll
        for (int blk = 0; blk < kBoxes; ++blk) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_f16(d, a0 + static_cast<uint64_t>((blk * kQBlock + k * 32) >> 4),
                        b0 + static_cast<uint64_t>((blk * kBoxBytes + k * 32) >> 4), kIdescQK, (blk | k) != 0);
        }
        tc::mma_commit(&sfull[sb]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) ok = issue_pv(nch - 1);
      if (!ok) {
        record_error(a.status, LSA_ERR_TIMEOUT, r, 11);
        *abort_flag = 1;
      }
      // every MMA issued must finish before TMEM is released
      tc::mma_commit(done);
      tc::mbar_wait(done, 0, nullptr);
      // the last chunk buffers' releases are asynchronous arrivals that must
      // land before the barriers are invalidated
      if (ok)
        for (int i = nch > kNBuf ? nch - kNBuf : 0; i < nch; ++i)
          tc::mbar_wait(&kvempty[i % kNBuf], static_cast<uint32_t>((i / kNBuf) & 1), abort_flag);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int quarter = warp & 3;                       // TMEM lanes 32q .. 32q+31
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    const bool srow = lane < 16;                        // lanes holding a score row
    const int head_local = quarter * 16 + (lane & 15);  // 0..63
    const float c2 = a.scale * kLog2e;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    // validity of the chunk's rows (lane and lane + 32), looked up one chunk ahead
    auto valid2 = [&](int jj, bool* x, bool* y) {
      const int jl[2] = {jj < nch ? j0 + jj * kChunk + lane : j1, jj < nch ? j0 + jj * kChunk + 32 + lane : j1};
      int64_t rr[2];
      entry_rows<2>(a, ad, rc, r, jl, j1, false, rr);
      *x = rr[0] >= 0;
      *y = rr[1] >= 0;
    };
    bool va, vb;
    valid2(0, &va, &vb);
    for (int j = 0; j < nch; ++j) {
      const int sb = j & 1;
      const uint32_t mlo = __ballot_sync(0xffffffffu, va), mhi = __ballot_sync(0xffffffffu, vb);
      if (j + 1 < nch) valid2(j + 1, &va, &vb);
      if (!tc::mbar_wait(&sfull[sb], (j >> 1) & 1, abort_flag)) { ok = false; break; }
      tc::tc_fence_after();
      float s[64];
      {
        float t0[32], t1[32];
        tc::tmem_ld32(tmem + lane_base + kColS + sb * kChunk, t0);
        tc::tmem_ld32(tmem + lane_base + kColS + sb * kChunk + 32, t1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = t0[i];
          s[32 + i] = t1[i];
        }
      }
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&sempty[sb]);
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        const bool valid = (i < 32) ? ((mlo >> i) & 1u) : ((mhi >> (i - 32)) & 1u);
        s[i] = valid ? s[i] * c2 : -INFINITY;
        mx = fmaxf(mx, s[i]);
      }
      const float m_new = fmaxf(m_run, mx);
      const bool need = srow && (j > 0) && (m_new > m_run + kRescaleLog2);
      if (__any_sync(0xffffffffu, need)) {
        // a rescale touches O: P V of chunk j-1 must have finished
        if (!tc::mbar_wait(pvdone, (j - 1) & 1, abort_flag)) { ok = false; break; }
        const float alpha_own = need ? ex2(m_run - m_new) : 1.f;
        const float alpha = __shfl_sync(0xffffffffu, alpha_own, lane & 15);
        tc::tc_fence_after();
#pragma unroll 1
        for (int cb = 0; cb < 8; ++cb) {
          float v[32];
          tc::tmem_ld32(tmem + lane_base + cb * 32, v);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha;
          tmem_st32(tmem + lane_base + cb * 32, v);
        }
        tmem_wait_st();
        if (need) {
          l *= alpha_own;
          m_run = m_new;
        }
      }
      if (j == 0) m_run = m_new;
      // probabilities (base 2): masked entries are -inf and give 2^-inf = 0; a
      // head with no valid entry yet (m_run = -inf) gives 0 everywhere.  P is
      // stored in bf16 and the row sum adds the rounded values.
      if (srow) {
        const float mref = m_run == -INFINITY ? INFINITY : m_run;
        float lsum[2] = {0.f, 0.f};
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          uint32_t w[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int i0 = c * 8 + 2 * u;
            const __nv_bfloat162 pb = __floats2bfloat162_rn(ex2(s[i0] - mref), ex2(s[i0 + 1] - mref));
            const float2 pf = __bfloat1622float2(pb);
            lsum[u & 1] += pf.x + pf.y;
            w[u] = *reinterpret_cast<const uint32_t*>(&pb);
          }
          *reinterpret_cast<uint4*>(kvs + (j % kNBuf) * kKvBytes + kRopeBox * kBoxBytes +
                                    tc::sw128_offset(head_local, c)) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        l += lsum[0] + lsum[1];
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(pfull);
    }
    if (!ok && lane == 0) {
      record_error(a.status, LSA_ERR_TIMEOUT, r, 12);
      *abort_flag = 1;
    }
    // final: wait for the last PV, normalise, store (bf16 output or fp32 partial)
    // A parity wait names a phase unambiguously only while the phase before it
    // has completed.  The last score commit this warp waited for precedes the
    // issue of P V(nch-2), so that phase is waited for first, then P V(nch-1).
    bool fin = ok;
    if (ok && nch > 1) fin = tc::mbar_wait(pvdone, (nch - 2) & 1, abort_flag);
    if (fin && nch > 0) fin = tc::mbar_wait(pvdone, (nch - 1) & 1, abort_flag);
    const float l_h = __shfl_sync(0xffffffffu, l, lane & 15);
    const float m_h = __shfl_sync(0xffffffffu, m_run, lane & 15);
    const float inv = l_h > 0.f ? 1.f / l_h : 0.f;
    const float lse = l_h > 0.f ? (m_h + log2f(l_h)) * kLn2 : -INFINITY;
    const int h = half * kHeadsCta + head_local;
    const int dim0 = lane < 16 ? 0 : 256;
    if (fin) tc::tc_fence_after();
#pragma unroll 1
    for (int cb = 0; cb < 8; ++cb) {
      float v[32];
      if (fin && nch > 0) {
        tc::tmem_ld32(tmem + lane_base + cb * 32, v);
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (P.nsplit == 1) {
        store_bf16x32(reinterpret_cast<__nv_bfloat16*>(a.out) + (static_cast<int64_t>(r) * kHeadsAll + h) * kDv +
                          dim0 + cb * 32, v, inv);
      } else {
        float* o = P.part_o + ((static_cast<int64_t>(r) * P.nsplit + split) * kHeadsAll + h) * kDv + dim0 + cb * 32;
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<float4*>(o + 4 * u) =
              make_float4(v[4 * u] * inv, v[4 * u + 1] * inv, v[4 * u + 2] * inv, v[4 * u + 3] * inv);
      }
    }
    if (lane < 16) {
      if (P.nsplit == 1) {
        if (a.lse) a.lse[static_cast<int64_t>(r) * kHeadsAll + h] = lse;
      } else {
        P.part_lse[(static_cast<int64_t>(r) * P.nsplit + split) * kHeadsAll + h] = lse;
      }
    }
  }
  // ---------------------------------------------------------------- split merge by the last CTA
  if (P.nsplit > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const int prev = atomicAdd(P.counters + 2 * r + half, 1);
      *last_flag = prev == P.nsplit - 1;
    }
    __syncthreads();
    if (*last_flag) {
      __threadfence();
      if (threadIdx.x == 0) P.counters[2 * r + half] = 0;  // left zeroed for the next call
      // weights of every split for the 64 heads
      float* wsm = reinterpret_cast<float*>(kvs);         // [nsplit][64] in the idle chunk buffer, nsplit <= 32
      const int ns = P.nsplit;
      const float* lse_p = P.part_lse + static_cast<int64_t>(r) * ns * kHeadsAll + half * kHeadsCta;
      if (threadIdx.x < kHeadsCta) {
        const int hl = threadIdx.x;
        float mx = -INFINITY;
        for (int sp = 0; sp < ns; ++sp) mx = fmaxf(mx, __ldcg(lse_p + sp * kHeadsAll + hl));
        float den = 0.f;
        for (int sp = 0; sp < ns; ++sp) {
          const float e = mx == -INFINITY ? 0.f : exp2f((__ldcg(lse_p + sp * kHeadsAll + hl) - mx) * kLog2e);
          wsm[sp * kHeadsCta + hl] = e;
          den += e;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        for (int sp = 0; sp < ns; ++sp) wsm[sp * kHeadsCta + hl] *= inv;
        if (a.lse) a.lse[static_cast<int64_t>(r) * kHeadsAll + half * kHeadsCta + hl] = den > 0.f ? mx + logf(den) : -INFINITY;
      }
      __syncthreads();
      // 64 heads x 128 groups of 4 dims over every thread of the CTA, eight
      // groups per pass with the loads of two splits in flight together
      const float4* po = reinterpret_cast<const float4*>(P.part_o);
      constexpr int kItems = kHeadsCta * (kDv / 4);
      for (int it0 = threadIdx.x; it0 < kItems; it0 += 8 * kThreads) {
        float4 acc[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int sp0 = 0; sp0 < ns; sp0 += 2) {
          float4 x[8][2];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int item = it0 + u * kThreads;
            const int hl = item / (kDv / 4), c4 = item % (kDv / 4);
            const int h = half * kHeadsCta + hl;
#pragma unroll
            for (int v = 0; v < 2; ++v)
              x[u][v] = (item < kItems && sp0 + v < ns)
                            ? __ldcg(po + ((static_cast<int64_t>(r) * ns + sp0 + v) * kHeadsAll + h) * (kDv / 4) + c4)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int item = it0 + u * kThreads;
            const int hl = (item < kItems ? item : 0) / (kDv / 4);
#pragma unroll
            for (int v = 0; v < 2; ++v) {
              const float wgt = sp0 + v < ns ? wsm[(sp0 + v) * kHeadsCta + hl] : 0.f;
              acc[u].x = fmaf(wgt, x[u][v].x, acc[u].x); acc[u].y = fmaf(wgt, x[u][v].y, acc[u].y);
              acc[u].z = fmaf(wgt, x[u][v].z, acc[u].z); acc[u].w = fmaf(wgt, x[u][v].w, acc[u].w);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int item = it0 + u * kThreads;
          if (item >= kItems) continue;
          const int hl = item / (kDv / 4), c4 = item % (kDv / 4);
          const int h = half * kHeadsCta + hl;
          const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y), hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t*>(&lo);
          pk.y = *reinterpret_cast<const uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                    (static_cast<int64_t>(r) * kHeadsAll + h) * kDv + c4 * 4) = pk;
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    for (uint64_t* b = bars; b <= done; ++b) tc::mbar_inval(b);
  }
  __syncthreads();
}

// Splits of each row's selection: one wave of (split, half, row) CTAs, at most
// 32 (the merge keeps one weight per split and head in a chunk buffer).
inline int tc_nsplit(int32_t rows, int32_t k) {
  const int chunks = (k + kChunk - 1) / kChunk;
  const int64_t per = 2LL * (rows > 0 ? rows : 1);       // CTAs per split
  int want = static_cast<int>(kPlanSMs / per);          // stay within one wave
  if (want > chunks) want = chunks;
  if (want > 32) want = 32;                              // merge weights fit one P buffer
  if (want < 1) want = 1;
  const int cps = (chunks + want - 1) / want;            // equal chunks per split
  return (chunks + cps - 1) / cps;
}

}  // namespace attn
}  // namespace lsa
