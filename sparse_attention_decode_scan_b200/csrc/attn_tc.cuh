#pragma once
// Sparse MQA decode on the sm_100a tensor cores (tcgen05 + TMEM), gathering
// the selected KV rows through the block table.
//
// The layer attends only the k tokens the lightning indexer kept (MLI abstract,
// sentence 2): o[h] = softmax_j(scale * q[h] . KV[idx_j]) . KV[idx_j][:512]
// over 128 query heads sharing 576-wide bf16 KV rows (value = first 512
// columns), plus lse[h].  Only the kept rows are read (the LeanSparse episode
// page: sparsity saves bytes read, the cache itself stays whole).
//
// Work: one CTA per (query row, half of the heads, split of the index list).
// 64 heads make the MMA's M side (M = 64), which uses lanes 0-15 or 16-31 of
// each 32-lane TMEM quarter: the query Q[64 x 576] (the score MMA's A operand,
// read from TMEM) and the scores S[64 x 64] sit on lanes 0-15, the fp32 output
// accumulator O[64 x 512] on lanes 16-31.
//   warps 0-3  producer: resolves the KV rows of the split's list entries into
//              a shared-memory table before the first gather, then gathers 64
//              rows per chunk with cp.async into the 128-byte-swizzled operand
//              layout (three chunk buffers; the chunk two ahead is prefetched
//              into L2) and publishes which rows exist
//   warp 4     MMA issuer: S = Q K^T (36 x M64N64K16, A from TMEM), O += P V
//              (8 x M64N256K16, V read MN-major from the same tile as K)
//   warps 5-8  load Q into TMEM, then the online softmax (base 2, lazy rescale
//              when the max grows by > 8): P[64 heads x 64 rows] is written
//              over the chunk's rope block (dims 512-575, dead once S is
//              computed), so P is buffered with the chunks
// (Below N = 64 an MMA costs as much as at N = 64 on this part, so 64-row
// chunks halve the score MMAs per row compared with 32-row chunks.)
// With several splits per row, each CTA writes a normalised partial and its
// lse; the split CTAs of a (row, half) then meet (co-resident by a cooperative
// launch) and each merges one slice, or a separate merge launch follows.
#include <math.h>

#include "common.cuh"
#include "internal.h"
#include "tc.cuh"
#include "topk_sel.cuh"

namespace lsa {
namespace attn {

constexpr int kHeadsAll = 128;
constexpr int kHeadsCta = 64;
constexpr int kD = 576;
constexpr int kDv = 512;
constexpr int kChunk = 64;                 // KV rows per chunk
constexpr int kNBuf = 3;                   // chunk buffers
constexpr int kBoxes = kD / 64;            // 9 column blocks of 64 dims
constexpr int kBoxBytes = kChunk * 128;    // 64 rows x 128 B
constexpr int kKvBytes = kBoxes * kBoxBytes;          // 73728
constexpr int kRowTab = 2048;                         // KV rows of up to 2048 list entries, resolved ahead in smem
constexpr int kRopeBox = kBoxes - 1;                  // column block of dims 512-575; holds P after S
constexpr int kThreads = 288;
constexpr int kProdThreads = 128;
constexpr int kWarpMma = 4;                // warps 5-8: softmax
constexpr int kSmemBytes = kNBuf * kKvBytes + kRowTab * 4 + 1024 /*barriers*/ + 1024 /*align*/;
// TMEM (512 columns x 128 lanes; an M = 64 tile uses lanes 0-15 or 16-31 of
// each 32-lane quarter):
//   lanes 0-15:  Q, dims 0-575 as bf16 pairs, the QK MMA's A operand (columns
//                0-287) | S (columns 288-351)
//   lanes 16-31: O, dims 0-511 (columns 0-511)
// An A operand in TMEM must start at lane 0 and its accumulator must sit on
// the same lanes, so Q and S share lanes 0-15.  Shared memory then holds three
// chunk buffers and a table of the split's KV rows.
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColQ = 0;              // Q dims 0-575 (lane offset 0)
constexpr uint32_t kColS = 288;            // S (lane offset 0)
constexpr uint32_t kLaneHi = 16u << 16;    // TMEM address offset of lane 16 (O)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.f;        // lazy rescale threshold (factor 256)

constexpr uint32_t kIdescQK = tc::idesc(tc::kFmtBF16, tc::kFmtBF16, 64, kChunk);
constexpr uint32_t kIdescPV = tc::idesc(tc::kFmtBF16, tc::kFmtBF16, 64, 256) | (1u << 16);  // B MN-major

static_assert(kSmemBytes <= 232448, "shared memory");

// How the split partials of a (row, 64 heads) are combined.
constexpr int kMergeSeparate = 0;  // partials only; a separate merge launch follows
constexpr int kMergeInKernel = 1;  // the split CTAs meet, then each merges a slice
constexpr int kMergeCluster = 2;   // the split CTAs of a (row, half) form a cluster and merge through DSMEM
                                   // (needs every CTA resident at once)

struct TcAttnParams {
  AttnArgs a;
  int nsplit;
  int split_len;   // multiple of kChunk
  float* part_o;   // [rows][nsplit][128][512]
  float* part_lse; // [rows][nsplit][128]
  int* counters;   // [rows][2], zeroed before the launch (kMergeInKernel)
  int merge;       // kMergeSeparate, kMergeInKernel or kMergeCluster
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

// D[tmem] (+)= A[tmem] * B[smem]^T, kind::f16 (A read from tensor memory).
__device__ __forceinline__ void mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
      "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
      "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
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

// KV rows of the list entries at offsets [lo, hi) of the split (list = the
// row's selection from the split's first entry, in global memory, or in shared
// memory with list_shared, where it may be rtab itself) into rtab[e - base],
// by n threads (tid): per pass 8 list loads in flight, then their 8
// block-table loads.  -1 marks padding, positions out of range and bad blocks (reported
// when `report`).  Out of line: it runs once per table part, and one compact
// copy is cheaper to fetch than inlined ones.
static __device__ __noinline__ void fill_rows(const int32_t* list, const int32_t* bt, int32_t max_blocks, int32_t block_size,
                                              int64_t n_blocks, int64_t row_base, int64_t L, bool ok, DevStatus* status,
                                              int r, int base, int lo, int hi, int tid, int n, bool report,
                                              int32_t* rtab, bool list_shared = false) {
  const bool paged = block_size > 0;
  const DivU32 bs = make_divu32(paged ? static_cast<uint32_t>(block_size) : 1u);
  for (int e = lo + tid; e < hi; e += 8 * n) {
    int32_t pos[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int eu = e + u * n;
      // L2-coherent load: in the fused step the selection is written earlier in the same launch
      pos[u] = (eu < hi && ok) ? (list_shared ? list[eu] : __ldcg(list + eu)) : -1;
    }
    int32_t blk[8];
    uint32_t lb[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      blk[u] = -1;
      lb[u] = 0;
      if (paged && pos[u] >= 0 && pos[u] < L) {
        lb[u] = divu32(bs, static_cast<uint32_t>(pos[u]));
        if (lb[u] < static_cast<uint32_t>(max_blocks)) blk[u] = __ldg(bt + lb[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int eu = e + u * n;
      int64_t row = -1;
      if (!paged) {
        if (pos[u] >= 0 && pos[u] < L) row = row_base + pos[u];
      } else if (blk[u] >= 0 && blk[u] < n_blocks) {
        row = static_cast<int64_t>(blk[u]) * block_size + (pos[u] - static_cast<int32_t>(lb[u] * bs.d));
      }
      if (report && pos[u] >= 0 && row < 0) record_error(status, LSA_ERR_BOUNDS, r, pos[u]);
      if (eu < hi) rtab[eu - base] = static_cast<int32_t>(row);
    }
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

// Merge weights of the heads [hl0, hl1) of one (row, half): the ns split lse
// values (load(s, hl)) are gathered into wsm[s][hl] by one thread per pair,
// then one thread per head turns them into w[s][hl] = exp(lse_s - m) /
// sum_s' exp(lse_s' - m), m the largest, the sum taken in ascending split
// order; the slice that holds a head's first group (hl * 128 >= i0) also
// writes the head's merged lse to lse_row[hl].  The loops are kept rolled:
// this code runs once per CTA, on a cold instruction cache.
template <class Load>
__device__ __forceinline__ void merge_weights(int ns, int hl0, int hl1, int i0, Load load, float* wsm,
                                              float* lse_row) {
  const int nh = hl1 - hl0;
  for (int i = static_cast<int>(threadIdx.x); i < ns * nh; i += kThreads) {
    const int s = i / nh, hl = hl0 + i % nh;
    wsm[s * kHeadsCta + hl] = load(s, hl);
  }
  __syncthreads();
  for (int hl = hl0 + static_cast<int>(threadIdx.x); hl < hl1; hl += kThreads) {
    float mx = -INFINITY;
#pragma unroll 1
    for (int s = 0; s < ns; ++s) mx = fmaxf(mx, wsm[s * kHeadsCta + hl]);
    float den = 0.f;
#pragma unroll 1
    for (int s = 0; s < ns; ++s) {
      const float e = mx != -INFINITY ? exp2f((wsm[s * kHeadsCta + hl] - mx) * kLog2e) : 0.f;
      wsm[s * kHeadsCta + hl] = e;
      den += e;
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
#pragma unroll 1
    for (int s = 0; s < ns; ++s) wsm[s * kHeadsCta + hl] *= inv;
    if (lse_row && hl * (kDv / 4) >= i0) lse_row[hl] = den > 0.f ? mx + logf(den) : -INFINITY;
  }
}

// out[r][half*64 + g/128][4(g%128) .. +3] = sum_s w[s][head] * part_o[r][s][..]
// for the groups g in [i0, i1) of one (row, half), U groups per thread and
// pass with the loads of V splits in flight together; w in shared memory
// ([nsplit][64], normalised), splits summed in ascending order.
template <int U, int V>
__device__ __forceinline__ void merge_slice(const TcAttnParams& P, int r, int half, int i0, int i1,
                                            const float* wsm) {
  const int ns = P.nsplit;
  const float4* po = reinterpret_cast<const float4*>(P.part_o);
  for (int it0 = i0 + threadIdx.x; it0 < i1; it0 += U * kThreads) {
    float4 acc[U];
#pragma unroll
    for (int u = 0; u < U; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sp0 = 0; sp0 < ns; sp0 += V) {
      float4 x[U][V];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int item = it0 + u * kThreads;
        const int hl = item / (kDv / 4), c4 = item % (kDv / 4);
        const int h = half * kHeadsCta + hl;
#pragma unroll
        for (int v = 0; v < V; ++v)
          x[u][v] = (item < i1 && sp0 + v < ns)
                        ? __ldcg(po + ((static_cast<int64_t>(r) * ns + sp0 + v) * kHeadsAll + h) * (kDv / 4) + c4)
                        : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int item = it0 + u * kThreads;
        const int hl = (item < i1 ? item : i0) / (kDv / 4);
#pragma unroll
        for (int v = 0; v < V; ++v) {
          const float wgt = sp0 + v < ns ? wsm[(sp0 + v) * kHeadsCta + hl] : 0.f;
          acc[u].x = fmaf(wgt, x[u][v].x, acc[u].x); acc[u].y = fmaf(wgt, x[u][v].y, acc[u].y);
          acc[u].z = fmaf(wgt, x[u][v].z, acc[u].z); acc[u].w = fmaf(wgt, x[u][v].w, acc[u].w);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int item = it0 + u * kThreads;
      if (item >= i1) continue;
      const int hl = item / (kDv / 4), c4 = item % (kDv / 4);
      const int h = half * kHeadsCta + hl;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y), hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t*>(&lo);
      pk.y = *reinterpret_cast<const uint32_t*>(&hi);
      *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(P.a.out) +
                                (static_cast<int64_t>(r) * kHeadsAll + h) * kDv + c4 * 4) = pk;
    }
  }
}

// Bounded wait (acquire) until *flag != 0; its value, or 0 after tc::kWaitLimitNs.
__device__ __forceinline__ uint32_t wait_value(const uint32_t* flag) {
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return v;
    if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) return 0;
    __nanosleep(64);
  }
}

// Entries [j0, j1) of a row's ordered selection (ascending positions) from the
// top-k's exact bitmap of the row and its per-segment first entries (segoff,
// keff at [nseg]), as positions (-1 past keff) into rtab[0, j1 - j0): only the
// segments holding those entries are compacted.  By the 128 producer threads
// (named barrier 4); scratch: 1 KB plus the staged words (padded per thread)
// at `scratch` + 1024.
static __device__ __noinline__ void split_entries(const uint32_t* segoff, const uint32_t* bitmap, int64_t nwords,
                                                  int nseg, int64_t seg_len, int j0, int j1, int32_t* rtab,
                                                  uint8_t* scratch, int t) {
  constexpr int NT = kProdThreads;
  int* warp_sums = reinterpret_cast<int*>(scratch);
  uint32_t* so = reinterpret_cast<uint32_t*>(scratch + 128);  // [nseg + 1]
  uint32_t* st = reinterpret_cast<uint32_t*>(scratch + 1024);
  for (int i = t; i <= nseg; i += NT) so[i] = __ldcg(segoff + i);
  asm volatile("bar.sync 4, %0;" ::"n"(NT) : "memory");
  const int keff = static_cast<int>(so[nseg]);
  const int n_ent = j1 - j0;
  const int e_hi = keff < j1 ? keff : j1;
  for (int e = (keff > j0 ? keff : j0) - j0 + t; e < n_ent; e += NT) rtab[e] = -1;
  if (j0 < e_hi) {
    // the segments holding entries j0 and e_hi - 1
    int s_lo = 0, s_hi = 0;
    for (int s2 = 0; s2 < nseg; ++s2) {
      if (static_cast<int>(so[s2]) <= j0) s_lo = s2;
      if (static_cast<int>(so[s2]) <= e_hi - 1) s_hi = s2;
    }
    const int64_t wps = seg_len / 32;
    const int64_t w_lo = s_lo * wps;
    const int64_t w_hi = (s_hi + 1) * wps < nwords ? (s_hi + 1) * wps : nwords;
    const int W = static_cast<int>(w_hi - w_lo);
    const int per = (W + NT - 1) / NT, stride = per | 1;
    const DivU32 dper = make_divu32(static_cast<uint32_t>(per));
    for (int w0 = t; w0 < W; w0 += 8 * NT) {
      uint32_t v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) v[u] = w0 + u * NT < W ? __ldcg(bitmap + w_lo + w0 + u * NT) : 0u;
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const uint32_t w = static_cast<uint32_t>(w0 + u * NT);
        if (w0 + u * NT < W) {
          const uint32_t q = divu32(dper, w);
          st[q * stride + (w - q * per)] = v[u];
        }
      }
    }
    asm volatile("bar.sync 4, %0;" ::"n"(NT) : "memory");
    const int wa = t * per;
    const int nm = W - wa < per ? (W - wa > 0 ? W - wa : 0) : per;
    int cnt = 0;
    for (int i = 0; i < nm; ++i) cnt += __popc(st[t * stride + i]);
    int tot;
    int o = static_cast<int>(so[s_lo]) + tk::tk_excl_scan<NT, 4>(cnt, warp_sums, &tot);
    for (int i = 0; i < nm && o < e_hi; ++i) {
      uint32_t x = st[t * stride + i];
      const int px = __popc(x);
      if (o + px <= j0) {
        o += px;
        continue;
      }
      while (x) {
        const int b = __ffs(x) - 1;
        x &= x - 1;
        if (o >= j0 && o < e_hi) rtab[o - j0] = static_cast<int32_t>((w_lo + wa + i) * 32 + b);
        ++o;
      }
    }
  }
  asm volatile("bar.sync 4, %0;" ::"n"(NT) : "memory");
}

// Bounded wait (acquire) until *flag != 0; false after tc::kWaitLimitNs.
__device__ __forceinline__ bool wait_flag(const uint32_t* flag) {
  const uint64_t t0 = tc::globaltimer_ns();
  for (;;) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(flag) : "memory");
    if (v != 0) return true;
    if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) return false;
    __nanosleep(64);
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
  uint8_t* kvs = smem;                                                  // kNBuf chunk buffers
  int32_t* rtab = reinterpret_cast<int32_t*>(kvs + kNBuf * kKvBytes);   // KV rows of the split's entries (-1: none)
  uint64_t* bars = reinterpret_cast<uint64_t*>(rtab + kRowTab);
  uint64_t* qfull = bars;
  uint64_t* kvfull = bars + 1;            // [kNBuf]
  uint64_t* kvempty = kvfull + kNBuf;     // [kNBuf]
  uint64_t* sfull = kvempty + kNBuf;      // S(j) computed
  uint64_t* rdone = sfull + 1;            // S(j) read and O rescaled: S(j+1) may be computed
  uint64_t* pfull = rdone + 1;
  uint64_t* pvdone = pfull + 1;
  uint64_t* done = pvdone + 1;
  uint64_t* vfull = done + 1;             // [kNBuf] the chunk's row validity is written
  uint64_t* mready = vfull + kNBuf;       // cluster merge: every split CTA has staged its partial
  uint64_t* mdone = mready + 1;           // cluster merge: every split CTA has read the others' partials
  uint64_t* bars_end = mdone + 1;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(bars_end);
  int* last_flag = const_cast<int*>(abort_flag) + 1;
  uint8_t* vrow = reinterpret_cast<uint8_t*>(last_flag + 1);  // [kNBuf][kChunk]: 1 = the row has a KV row
  float* slse = reinterpret_cast<float*>(vrow + kNBuf * kChunk);  // [64] cluster merge: the partial's lse
  const bool cmerge = P.nsplit > 1 && P.merge == kMergeCluster;
  // the producer waits for this row's data itself (no wait for the kernel before)
  const bool handoff = a.row_ready != nullptr || a.split_sel;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = split * P.split_len;
  const int j1 = min(a.k, j0 + P.split_len);
  const int nch = j1 > j0 ? (j1 - j0 + kChunk - 1) / kChunk : 0;

  if (threadIdx.x == 0) {
    tc::mbar_init(qfull, 4);  // the softmax warps' TMEM stores of Q
    for (int i = 0; i < kNBuf; ++i) {
      tc::mbar_init(&kvfull[i], kProdThreads);
      tc::mbar_init(&kvempty[i], 1);
    }
    tc::mbar_init(sfull, 1);
    tc::mbar_init(rdone, 4);
    tc::mbar_init(pfull, 4);
    tc::mbar_init(pvdone, 1);
    tc::mbar_init(done, 1);
    for (int i = 0; i < kNBuf; ++i) tc::mbar_init(&vfull[i], 4);  // one arrival per producer warp
    tc::mbar_init(mready, cmerge ? P.nsplit : 1);                   // one arrival per split CTA
    tc::mbar_init(mdone, cmerge ? P.nsplit : 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  __syncthreads();
  if (cmerge) tc::cluster_arrive_relaxed();  // waited for before the first remote arrival
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
    // The KV rows of the split's list entries are resolved ahead into a table
    // in shared memory (up to kRowTab entries at a time), so the gather loop
    // issues no dependent global load of its own.  The first part is resolved
    // before the first gather: its two dependent rounds of loads (list, then
    // block table) cost about the same for 64 entries as for 2048, and HBM is
    // still idle then.
    const int n_ent = j1 - j0;
    const int32_t* bt = ad.block_size > 0 ? ad.block_table + static_cast<int64_t>(rc.b) * ad.max_blocks : nullptr;
    auto fill_table = [&](int e0) {  // entries [e0, e0 + kRowTab)
      const int hi = n_ent - e0 < kRowTab ? n_ent : e0 + kRowTab;
      fill_rows(a.idx + static_cast<int64_t>(r) * a.k + j0, bt, ad.max_blocks, ad.block_size, ad.n_blocks,
                static_cast<int64_t>(rc.b) * ad.max_len, rc.L, rc.ok, a.status, r, e0, e0, hi, t, kProdThreads,
                half == 0, rtab);
      asm volatile("bar.sync 4, %0;" ::"n"(kProdThreads) : "memory");  // the producer warps
    };
    auto row_of = [&](int jj, int m) -> int64_t {  // chunk jj, this thread's m-th row
      const int e = jj * kChunk + rbase + 16 * m;  // entry offset in the split
      return jj < nch ? static_cast<int64_t>(rtab[e % kRowTab]) : -1;
    };
    auto prefetch_l2 = [&](int jj, int j_now) {
      // only chunks whose rows are in the table now
      if (sub != 0 || jj >= nch || (jj * kChunk) / kRowTab != (j_now * kChunk) / kRowTab) return;
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int64_t row = row_of(jj, m);
        if (row >= 0)
          asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(
                           reinterpret_cast<const uint8_t*>(a.cache.kv) + row * (kD * 2)),
                       "r"(kD * 2)
                       : "memory");
      }
    };
    uint32_t sel_state = 2;  // 2: the row's selection is in a.idx
    if (a.split_sel) {
      // decode step, launched early: wait for the top-k's split select of this
      // row (1: exact bitmap and segment offsets, 2: the full selection in idx)
      const tk::TkLayout TL = tk::tk_layout(a.tk_ws, a.rows, a.tk_ncols);
      if (t == 0) {
        const uint32_t v = wait_value(TL.selready + r);
        if (v == 0) {
          record_error(a.status, LSA_ERR_TIMEOUT, r, 22);
          *abort_flag = 1;
        }
        *last_flag = static_cast<int>(v);
      }
      asm volatile("bar.sync 4, %0;" ::"n"(kProdThreads) : "memory");  // the producer warps
      sel_state = static_cast<uint32_t>(*last_flag);
      if (sel_state == 1) {
        // this split's entries, compacted from the segments that hold them
        // (the chunk buffers are idle until the first gather)
        split_entries(TL.segoff + static_cast<int64_t>(r) * (tk::kMaxSeg + 1),
                      TL.bitmap + static_cast<int64_t>(r) * TL.words, TL.words, a.tk_nseg, a.tk_seg_len, j0, j1, rtab,
                      kvs, t);
        if (a.idx_w && half == 0)
          for (int e = t; e < n_ent; e += kProdThreads) a.idx_w[static_cast<int64_t>(r) * a.k + j0 + e] = rtab[e];
        fill_rows(rtab, bt, ad.max_blocks, ad.block_size, ad.n_blocks, static_cast<int64_t>(rc.b) * ad.max_len, rc.L,
                  rc.ok, a.status, r, 0, 0, n_ent, t, kProdThreads, half == 0, rtab, true);
        asm volatile("bar.sync 4, %0;" ::"n"(kProdThreads) : "memory");  // the producer warps
      } else if (sel_state == 0) {
        for (int e = t; e < kRowTab; e += kProdThreads) rtab[e] = -1;
        asm volatile("bar.sync 4, %0;" ::"n"(kProdThreads) : "memory");  // the producer warps
      }
    } else if (a.row_ready) {
      // decode step, launched early: wait for this row's selection only
      if (t == 0 && !wait_flag(a.row_ready + r)) {
        record_error(a.status, LSA_ERR_TIMEOUT, r, 21);
        *abort_flag = 1;
      }
      asm volatile("bar.sync 4, %0;" ::"n"(kProdThreads) : "memory");  // the producer warps
    } else {
      tc::griddep_wait();  // launched early in a decode step: the selection is complete from here on
    }
    if (sel_state == 2) fill_table(0);
    prefetch_l2(0, 0);
    prefetch_l2(1, 0);
#pragma unroll 1
    for (int j = 0; j < nch; ++j) {
      const int b = j % kNBuf;
      if (j > 0 && (j * kChunk) % kRowTab == 0) {  // the next kRowTab entries (splits longer than the table)
        // every producer thread has read its rows of the previous part
        asm volatile("bar.sync 4, %0;" ::"n"(kProdThreads) : "memory");
        fill_table(j * kChunk);
        prefetch_l2(j, j);
        prefetch_l2(j + 1, j);
      }
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
      int64_t R0[4];
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int i = rbase + 16 * m;
        R0[m] = row_of(j, m);
        if (R0[m] >= 0) {
          const uint8_t* src = reinterpret_cast<const uint8_t*>(a.cache.kv) + R0[m] * (kD * 2);
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
      // the softmax masks the rows without a KV row
      if (sub == 0) {
#pragma unroll
        for (int m = 0; m < 4; ++m) vrow[b * kChunk + rbase + 16 * m] = R0[m] >= 0 ? 1 : 0;
      }
      __syncwarp();
      if ((t & 31) == 0) tc::mbar_arrive(&vfull[b]);
      prefetch_l2(j + 2, j);
    }
    asm volatile("cp.async.wait_all;" ::: "memory");
  } else if (warp == kWarpMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (!handoff) tc::griddep_wait();
    if (lane == 0 && nch > 0) {
      bool ok = tc::mbar_wait(qfull, 0, abort_flag);
      tc::fence_proxy_async_smem();
      tc::tc_fence_after();  // Q's TMEM part was stored by the softmax warps
      // Two event streams, served as they become ready: S(j) = Q K(j)^T once
      // chunk j has landed and its score buffer is free, and P V(i) once P(i)
      // is written.  P V(i) goes out as soon as it can (not after S(i+1)), so
      // chunk i's buffer is released while chunk i+1 is still arriving and two
      // gathers overlap.  S(j) waits until P V(j-2) has been issued: its commit
      // then covers P V(j-2), which the softmax's parity wait on P V(j-1) needs.
      int next_s = 0, next_pv = 0;
      uint64_t t_last = tc::globaltimer_ns();
      uint32_t spin = 0;
      while (ok && next_pv < nch) {
        bool progressed = false;
        if (next_pv < next_s && tc::mbar_test(pfull, static_cast<uint32_t>(next_pv & 1))) {
          const int i = next_pv;
          tc::tc_fence_after();
          const uint32_t kv_u = tc::smem_u32(kvs + (i % kNBuf) * kKvBytes);
          const uint32_t p_u = kv_u + kRopeBox * kBoxBytes;  // P(i) sits in chunk i's rope block
          const uint64_t pa0 = tc::desc_sw128(p_u), vb0 = desc_sw128_mn(kv_u, kBoxBytes);
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const uint32_t d = tmem + kLaneHi + 256u * c;  // O dims 256c.. at columns 256c..
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk)
              tc::mma_f16(d, pa0 + static_cast<uint64_t>((kk * 32) >> 4),
                          vb0 + static_cast<uint64_t>(((4 * c) * kBoxBytes + kk * 2048) >> 4), kIdescPV,
                          (i > 0 || kk > 0) ? 1u : 0u);
          }
          tc::mma_commit(pvdone);
          tc::mma_commit(&kvempty[i % kNBuf]);
          ++next_pv;
          progressed = true;
        }
        // S(j) also waits until the softmax has read S(j-1) (one S buffer) and
        // finished any rescale of O, which rewrites the Q and S lanes as well:
        // no MMA may touch TMEM meanwhile.
        if (next_s < nch && next_s <= next_pv + 1) {
          const int j = next_s;
          const int b = j % kNBuf;
          if (tc::mbar_test(&kvfull[b], static_cast<uint32_t>((j / kNBuf) & 1)) &&
              (j == 0 || tc::mbar_test(rdone, static_cast<uint32_t>((j - 1) & 1)))) {
            tc::fence_proxy_async_smem();
            tc::tc_fence_after();
            const uint32_t d = tmem + kColS;
            // descriptors of the 36 K-steps differ only in the start-address field
            // (addresses stay below 256 KB, so the 14-bit field never carries)
            const uint64_t b0 = tc::desc_sw128(tc::smem_u32(kvs + b * kKvBytes));
            // Q from TMEM, 16 dims = 8 columns per K-step
#pragma unroll
            for (int blk = 0; blk < kBoxes; ++blk) {
#pragma unroll
              for (int k = 0; k < 4; ++k)
                mma_f16_ta(d, tmem + kColQ + static_cast<uint32_t>((blk * 4 + k) * 8),
                           b0 + static_cast<uint64_t>((blk * kBoxBytes + k * 32) >> 4), kIdescQK, (blk | k) != 0);
            }
            tc::mma_commit(sfull);
            ++next_s;
            progressed = true;
          }
        }
        if (progressed) {
          t_last = tc::globaltimer_ns();
        } else if ((++spin & 63u) == 0) {
          if (*abort_flag || tc::globaltimer_ns() - t_last > tc::kWaitLimitNs) ok = false;
        }
      }
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
    const bool srow = lane < 16;                        // lanes holding a score row; lanes 16-31 hold O rows
    const int head_local = quarter * 16 + (lane & 15);  // 0..63
    const int sl = lane & 15;                           // the score lane of this lane's head
    // Q (576 dims) of the heads of this quarter into TMEM lanes 0-15, columns
    // 0-287 (lanes 16-31 of those columns, O's, get zeros: the first P V
    // overwrites them).  In a decode step q is an input of the step, so it is
    // loaded while the top-k may still run.
    if (!a.q_early && !handoff) tc::griddep_wait();
    {
      const uint4* qsrc = reinterpret_cast<const uint4*>(
          reinterpret_cast<const uint8_t*>(a.q) +
          ((static_cast<int64_t>(r) * kHeadsAll + half * kHeadsCta + head_local) * kD) * 2);
#pragma unroll 1
      for (int g = 0; g < kBoxes; g += 3) {  // 64 dims = 32 columns per group, three groups of loads in flight
        uint4 x[24];
#pragma unroll
        for (int i = 0; i < 24; ++i) x[i] = lane < 16 ? __ldg(qsrc + g * 8 + i) : make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int gg = 0; gg < 3; ++gg) {
          uint32_t v[32];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            v[4 * i] = x[gg * 8 + i].x; v[4 * i + 1] = x[gg * 8 + i].y;
            v[4 * i + 2] = x[gg * 8 + i].z; v[4 * i + 3] = x[gg * 8 + i].w;
          }
          tmem_st32u(tmem + lane_base + kColQ + (g + gg) * 32, v);
        }
      }
      tmem_wait_st();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(qfull);
    }
    if (a.q_early && !handoff) tc::griddep_wait();
    const float c2 = a.scale * kLog2e;
    float m_run = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nch; ++j) {
      // validity of the chunk's rows lane and lane + 32, from the producer
      const int b = j % kNBuf;
      if (!tc::mbar_wait(&vfull[b], (j / kNBuf) & 1, abort_flag)) { ok = false; break; }
      const uint32_t mlo = __ballot_sync(0xffffffffu, vrow[b * kChunk + lane] != 0);
      const uint32_t mhi = __ballot_sync(0xffffffffu, vrow[b * kChunk + 32 + lane] != 0);
      if (!tc::mbar_wait(sfull, j & 1, abort_flag)) { ok = false; break; }
      tc::tc_fence_after();
      float s[64];
      {
        float t0[32], t1[32];
        tc::tmem_ld32(tmem + lane_base + kColS, t0);       // lanes 0-15: S rows
        tc::tmem_ld32(tmem + lane_base + kColS + 32, t1);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          s[i] = t0[i];
          s[32 + i] = t1[i];
        }
      }
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
        // a rescale touches O: P V of chunk j-1 must have finished.  The 32-lane
        // accesses also cover lanes 0-15 (Q, S), whose bits are written back
        // untouched; no MMA runs meanwhile (S(j+1) waits for rdone).
        if (!tc::mbar_wait(pvdone, (j - 1) & 1, abort_flag)) { ok = false; break; }
        const float alpha_own = need ? ex2(m_run - m_new) : 1.f;
        const float alpha = __shfl_sync(0xffffffffu, alpha_own, sl);
        tc::tc_fence_after();
#pragma unroll 1
        for (int cb = 0; cb < 16; ++cb) {
          float v[32];
          tc::tmem_ld32(tmem + lane_base + cb * 32, v);
          tc::tmem_wait_ld();
          if (!srow) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
          }
          tmem_st32(tmem + lane_base + cb * 32, v);
        }
        tmem_wait_st();
        if (need) {
          l *= alpha_own;
          m_run = m_new;
        }
      }
      // S(j) has been read and O rescaled: S(j+1) may be computed
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(rdone);
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
      // P(j) may only be published once the MMA issuer has taken P(j-1)
      // (P V(j-1) issued and done): S(j) can be issued before P V(j-1), so
      // without this wait pfull could complete phases j-1 and j before the
      // issuer tests it for j-1, its parity would read "not yet" and the
      // issuer would stall.  The wait names its phase unambiguously: S(j)'s
      // commit covered P V(j-2).  It rarely waits (P V(j-1) runs right after
      // S(j), while this chunk's softmax is still busy).
      if (j > 0 && !tc::mbar_wait(pvdone, (j - 1) & 1, abort_flag)) { ok = false; break; }
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
    const float l_h = __shfl_sync(0xffffffffu, l, sl);
    const float m_h = __shfl_sync(0xffffffffu, m_run, sl);
    const float inv = l_h > 0.f ? 1.f / l_h : 0.f;
    const float lse = l_h > 0.f ? (m_h + log2f(l_h)) * kLn2 : -INFINITY;
    const int h = half * kHeadsCta + head_local;
    if (fin) tc::tc_fence_after();
    // lanes 16-31 hold the O rows: dims 32 cb .. 32 cb + 31 in columns 32 cb ..
#pragma unroll 1
    for (int cb = 0; cb < 16; ++cb) {
      float v[32];
      if (fin && nch > 0) {
        tc::tmem_ld32(tmem + lane_base + cb * 32, v);
        tc::tmem_wait_ld();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
      }
      if (srow) {
        // lanes 0-15 hold Q and S here
      } else if (P.nsplit == 1) {
        store_bf16x32(reinterpret_cast<__nv_bfloat16*>(a.out) + (static_cast<int64_t>(r) * kHeadsAll + h) * kDv +
                          cb * 32, v, inv);
      } else {
        // Staged in the idle chunk buffers as [64 heads][512], the 16-byte
        // pieces of each 128-byte segment rotated by (head & 7) so that the
        // warp's rows spread over the banks; written out coalesced below.
        float* stg = reinterpret_cast<float*>(kvs);
#pragma unroll
        for (int u = 0; u < 8; ++u)
          *reinterpret_cast<float4*>(stg + head_local * kDv + cb * 32 + ((u ^ (head_local & 7)) << 2)) =
              make_float4(v[4 * u] * inv, v[4 * u + 1] * inv, v[4 * u + 2] * inv, v[4 * u + 3] * inv);
      }
    }
    if (lane < 16) {
      if (P.nsplit == 1) {
        if (a.lse) a.lse[static_cast<int64_t>(r) * kHeadsAll + h] = lse;
      } else if (cmerge) {
        slse[head_local] = lse;
      } else {
        P.part_lse[(static_cast<int64_t>(r) * P.nsplit + split) * kHeadsAll + h] = lse;
      }
    }
  }
  // ---------------------------------------------------------------- split partials out
  // The CTA's partial O block [64 heads][512] is contiguous in part_o: every
  // thread copies 16-byte pieces from the staging area, consecutive threads to
  // consecutive addresses (full-line writes that drain quickly).
  if (P.nsplit > 1 && !cmerge) {
    __syncthreads();
    const float4* stg4 = reinterpret_cast<const float4*>(kvs);
    float4* dst = reinterpret_cast<float4*>(
        P.part_o + ((static_cast<int64_t>(r) * P.nsplit + split) * kHeadsAll + half * kHeadsCta) * kDv);
    for (int i = threadIdx.x; i < kHeadsCta * (kDv / 4); i += kThreads) {
      const int hl = i >> 7, d4 = i & 127;
      dst[i] = stg4[hl * (kDv / 4) + (d4 & ~7) + ((d4 & 7) ^ (hl & 7))];
    }
  }
  // ---------------------------------------------------------------- split merge
  // Every split CTA of (row, half) publishes its partials and counts itself;
  // once all have (a bounded wait: the CTAs are co-resident), each merges its
  // own slice of the 64 heads x 128 groups of 4 dims, so the merge reads run
  // on all split CTAs at once.
  if (P.nsplit > 1 && P.merge == kMergeInKernel) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      int* ctr = P.counters + 2 * r + half;
      atomicAdd(ctr, 1);
      int go = 1;
      const uint64_t t0 = tc::globaltimer_ns();
      for (;;) {
        int v;
        asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(ctr) : "memory");
        if (v >= P.nsplit) break;
        if (tc::globaltimer_ns() - t0 > tc::kWaitLimitNs) {
          go = 0;
          record_error(a.status, LSA_ERR_TIMEOUT, r, 13);
          break;
        }
        __nanosleep(32);
      }
      *last_flag = go;
    }
    __syncthreads();
    if (*last_flag) {
      const int ns = P.nsplit;
      constexpr int kItems = kHeadsCta * (kDv / 4);
      const int per = (kItems + ns - 1) / ns;
      const int i0 = split * per;
      const int i1 = i0 + per < kItems ? i0 + per : kItems;
      // weights of every split for the heads this slice touches
      float* wsm = reinterpret_cast<float*>(kvs);  // [nsplit][64] in the idle chunk buffer, nsplit <= 32
      const float* lse_p = P.part_lse + static_cast<int64_t>(r) * ns * kHeadsAll + half * kHeadsCta;
      const int hl0 = i0 / (kDv / 4), hl1 = i1 > i0 ? (i1 - 1) / (kDv / 4) + 1 : hl0;
      merge_weights(
          ns, hl0, hl1, i0, [&](int s2, int hl) { return __ldcg(lse_p + s2 * kHeadsAll + hl); }, wsm,
          a.lse ? a.lse + static_cast<int64_t>(r) * kHeadsAll + half * kHeadsCta : nullptr);
      __syncthreads();
      // About 16 loads in flight per thread: 8 groups x 2 splits when the slice
      // is large (few splits), 1 group x 16 splits when it is small (many)
      if (i1 - i0 >= 4 * kThreads)
        merge_slice<8, 2>(P, r, half, i0, i1, wsm);
      else
        merge_slice<1, 16>(P, r, half, i0, i1, wsm);
    }
  }
  // ---------------------------------------------------------------- cluster merge
  // The split CTAs of a (row, half) are one cluster (CTA rank = split).  Each
  // staged its normalised partial O [64 heads][512] (rotated pieces, as above)
  // and lse in its own shared memory; once all have (remote arrivals on every
  // CTA's mready), each merges its slice of the 64 heads x 128 groups of 4
  // dims reading the partials through DSMEM, and keeps its shared memory until
  // every CTA has finished reading (mdone).
  if (cmerge) {
    __syncthreads();
    tc::cluster_wait();  // every CTA of the cluster has initialised its barriers
    const int ns = P.nsplit;
    if (threadIdx.x == 0) {
      tc::fence_acq_rel_cluster();
      const uint32_t mr = tc::smem_u32(mready);
      for (int s2 = 0; s2 < ns; ++s2) tc::mbar_arrive_cluster(tc::cluster_map(mr, static_cast<uint32_t>(s2)));
    }
    if (tc::mbar_wait_cluster(mready, 0)) {
      constexpr int kItems = kHeadsCta * (kDv / 4);
      const int per = (kItems + ns - 1) / ns;
      const int i0 = split * per;
      const int i1 = i0 + per < kItems ? i0 + per : kItems;
      // weights [nsplit][64] past the staged partial (which peers read)
      float* wsm = reinterpret_cast<float*>(kvs + kHeadsCta * kDv * 4);
      const int hl0 = i0 / (kDv / 4), hl1 = i1 > i0 ? (i1 - 1) / (kDv / 4) + 1 : hl0;
      const uint32_t slse_u = tc::smem_u32(slse);
      merge_weights(
          ns, hl0, hl1, i0,
          [&](int s2, int hl) {
            return tc::ld_cluster_f32(tc::cluster_map(slse_u, static_cast<uint32_t>(s2)) + static_cast<uint32_t>(hl) * 4u);
          },
          wsm, a.lse ? a.lse + static_cast<int64_t>(r) * kHeadsAll + half * kHeadsCta : nullptr);
      __syncthreads();
      const uint32_t stg_u = tc::smem_u32(kvs);
      constexpr int U = 4;  // groups per thread and pass, loads in flight together (more: longer cold code)
#pragma unroll 1
      for (int it0 = i0 + threadIdx.x; it0 < i1; it0 += U * kThreads) {
        float4 acc[U];
#pragma unroll
        for (int u = 0; u < U; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t off[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int item = it0 + u * kThreads;
          const int hl = item >> 7, c4 = item & 127;
          off[u] = static_cast<uint32_t>(hl * (kDv / 4) + (c4 & ~7) + ((c4 & 7) ^ (hl & 7))) * 16u;
        }
        // two splits per step: 2U loads in flight; the splits are summed in ascending order
#pragma unroll 1
        for (int s2 = 0; s2 < ns; s2 += 2) {
          // this CTA's own partial is read from its shared memory directly
          const int s3 = s2 + 1 < ns ? s2 + 1 : s2;
          const uint32_t pb0 = s2 == split ? stg_u : tc::cluster_map(stg_u, static_cast<uint32_t>(s2));
          const uint32_t pb1 = s3 == split ? stg_u : tc::cluster_map(stg_u, static_cast<uint32_t>(s3));
          float4 x0[U], x1[U];
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const bool in = it0 + u * kThreads < i1;
            x0[u] = !in ? make_float4(0.f, 0.f, 0.f, 0.f)
                        : (s2 == split ? tc::ld_shared_f4(pb0 + off[u]) : tc::ld_cluster_f4(pb0 + off[u]));
            x1[u] = !(in && s2 + 1 < ns) ? make_float4(0.f, 0.f, 0.f, 0.f)
                                         : (s3 == split ? tc::ld_shared_f4(pb1 + off[u]) : tc::ld_cluster_f4(pb1 + off[u]));
          }
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int item = it0 + u * kThreads;
            const int hl = (item < i1 ? item : i0) >> 7;
            const float w0 = wsm[s2 * kHeadsCta + hl];
            acc[u].x = fmaf(w0, x0[u].x, acc[u].x); acc[u].y = fmaf(w0, x0[u].y, acc[u].y);
            acc[u].z = fmaf(w0, x0[u].z, acc[u].z); acc[u].w = fmaf(w0, x0[u].w, acc[u].w);
            if (s2 + 1 < ns) {
              const float w1 = wsm[(s2 + 1) * kHeadsCta + hl];
              acc[u].x = fmaf(w1, x1[u].x, acc[u].x); acc[u].y = fmaf(w1, x1[u].y, acc[u].y);
              acc[u].z = fmaf(w1, x1[u].z, acc[u].z); acc[u].w = fmaf(w1, x1[u].w, acc[u].w);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int item = it0 + u * kThreads;
          if (item >= i1) continue;
          const int hl = item >> 7, c4 = item & 127;
          const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y);
          const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t*>(&lo);
          pk.y = *reinterpret_cast<const uint32_t*>(&hi);
          *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) +
                                    (static_cast<int64_t>(r) * kHeadsAll + half * kHeadsCta + hl) * kDv + c4 * 4) = pk;
        }
      }
    } else if (threadIdx.x == 0) {
      record_error(a.status, LSA_ERR_TIMEOUT, r, 15);
    }
    __syncthreads();  // this CTA's reads of the others' partials have completed
    if (threadIdx.x == 0) {
      const uint32_t md = tc::smem_u32(mdone);
      for (int s2 = 0; s2 < ns; ++s2) tc::mbar_arrive_cluster(tc::cluster_map(md, static_cast<uint32_t>(s2)));
    }
    if (!tc::mbar_wait_cluster(mdone, 0) && threadIdx.x == 0) record_error(a.status, LSA_ERR_TIMEOUT, r, 16);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    for (uint64_t* b = bars; b < bars_end; ++b) tc::mbar_inval(b);
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
