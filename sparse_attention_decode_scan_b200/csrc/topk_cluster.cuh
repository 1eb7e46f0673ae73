#pragma once
// Top-k of one row by one thread-block cluster (rows of up to kClMaxCols
// positions): the same exact selection as the collect + select bodies of
// topk_sel.cuh (the k best-scored tokens, MLI abstract, sentence 2; ties to
// the lower position, -inf and NaN never taken, positions ascending, then -1),
// with the row's work spread over the cluster's CTAs instead of ending in one.
//
// CTA s of the cluster owns segment s of the row.  It reads the row's
// first-digit histogram (key bits [31:20]) and finds the threshold bin b1,
// then collects its segment: keys above b1 become a bitmap in its own shared
// memory, keys inside b1 a local candidate list.  After a cluster barrier
// every CTA runs the radix select of the threshold key T on bits [19:0] over
// all CTAs' candidates, read through distributed shared memory (the lists are
// short: a bin holds a few hundred keys at these sizes), marks its own
// candidates above T into its bitmap and those equal to T into a tie bitmap,
// and publishes two counts.  After a second barrier each CTA knows the
// selection entries before its segment and the ties left to it (the lowest
// positions equal to T are taken first), and compacts its own segment into
// the output.  If any CTA's candidates overflow its list, T's lower digits are
// counted by every CTA from its own staged segment, the counts summed across
// the cluster through distributed shared memory, and each segment re-read
// from shared memory to mark.
#include "tc.cuh"
#include "topk_sel.cuh"

namespace lsa {
namespace tk {

constexpr int kClThreads = kCollectThreads;        // the round shape of tk_round_load
constexpr int kClMaxSeg = 16;                      // CTAs per cluster (above 8: a non-portable cluster size)
constexpr int kClPortableSeg = 8;
constexpr int64_t kClMaxCols = int64_t(1) << 19;   // longer rows take the collect + select bodies
constexpr int64_t kClMaxSegLen = 32768;            // positions a CTA stages in shared memory (128 KB)
// Threshold-bin keys a CTA keeps, by the cluster's largest size: every CTA
// gathers all CTAs' lists, so 16-CTA clusters keep half as many per CTA to
// stay within shared memory.  (A bin holds a few hundred keys of a row at
// these sizes; a longer list overflows into the whole-row path, still exact.)
__host__ __device__ constexpr int cl_cap(int maxseg) { return maxseg > kClPortableSeg ? 512 : 1024; }

struct ClHdr {
  uint32_t nc;  // keys of the threshold bin in the segment (> cl_cap: the list overflowed)
  uint32_t gt;  // selected keys above T in the segment
  uint32_t eq;  // keys equal to T in the segment
  uint32_t pad;
};
// the segment's scores follow the header: 16-byte loads and bulk copies need it aligned
static_assert(sizeof(ClHdr) % 16 == 0, "header size");

struct ClPlan {
  int nseg;
  int64_t seg_len;  // multiple of kColRound
};

// Segments of a row: up to max_seg CTAs (at most kClMaxSeg), at least one
// collect round (kColRound positions) each.  nseg = 0: the row needs more
// segments than max_seg to keep each within kClMaxSegLen.
__host__ __device__ inline ClPlan cl_plan(int64_t n_cols, int max_seg = kClMaxSeg) {
  ClPlan p;
  int64_t rounds = (n_cols + kColRound - 1) / kColRound;
  if (rounds < 1) rounds = 1;
  const int64_t cap = max_seg < kClMaxSeg ? (max_seg < 1 ? 1 : max_seg) : kClMaxSeg;
  if ((rounds + cap - 1) / cap * kColRound > kClMaxSegLen) {
    p.nseg = 0;
    p.seg_len = 0;
    return p;
  }
  const int64_t ns = rounds < cap ? rounds : cap;
  const int64_t per = (rounds + ns - 1) / ns;
  p.seg_len = per * kColRound;
  p.nseg = static_cast<int>((rounds + per - 1) / per);
  return p;
}

// Shared memory of the body: header | the segment's scores | the row's
// first-digit histogram | bitmap of the segment | tie bitmap | candidates |
// every CTA's candidate keys, gathered.  The bitmaps are padded per thread
// (tk_pad) so the ordered walk over each thread's own words hits distinct
// banks.
__host__ __device__ inline int cl_bm_words(int64_t seg_len) {
  const TkPad p = tk_pad(seg_len, kClThreads);
  return (kClThreads * p.stride + 3) / 4 * 4;
}

// Clusters of up to 8 CTAs run the MAXSEG = 8 body, larger ones MAXSEG = 16.
__host__ __device__ constexpr int cl_maxseg(int nseg) { return nseg > kClPortableSeg ? kClMaxSeg : kClPortableSeg; }

__host__ __device__ inline size_t cl_smem(int64_t seg_len, int nseg) {
  const int maxseg = cl_maxseg(nseg);
  const size_t cap = static_cast<size_t>(cl_cap(maxseg));
  return sizeof(ClHdr) + static_cast<size_t>(seg_len) * 4 + static_cast<size_t>(kB1) * 4 +
         2 * static_cast<size_t>(cl_bm_words(seg_len)) * 4 + cap * 8 + static_cast<size_t>(maxseg) * cap * 4;
}

// Row r, segment s of ns (CTA rank s of the row's cluster).  `live` false (a
// wait before it ran out): the CTA does no work but still takes part in the
// cluster barriers.  ID: named barrier of the CTA's threads.
template <int ID, int MAXSEG>
__device__ void tk_cluster_row(const TopkArgs& a, int r, int s, int ns, int64_t seg_len, uint8_t* dsm, TkScratch& S,
                               bool live) {
  constexpr int NT = kClThreads;
  constexpr int CAP = cl_cap(MAXSEG);
  const int t = threadIdx.x;
  const int lane = t & 31;
  const TkLayout L = tk_layout(a.ws, a.rows, a.n_cols);
  const TkPad pad = tk_pad(seg_len, NT);
  const int bm_words = cl_bm_words(seg_len);
  ClHdr* hdr = reinterpret_cast<ClHdr*>(dsm);
  float* seg = reinterpret_cast<float*>(dsm + sizeof(ClHdr));               // [seg_len]
  uint32_t* hsm = reinterpret_cast<uint32_t*>(seg + seg_len);               // [kB1]
  uint32_t* bm = hsm + kB1;
  uint32_t* tb = bm + bm_words;
  uint2* cs = reinterpret_cast<uint2*>(tb + bm_words);
  uint32_t* allk = reinterpret_cast<uint32_t*>(cs + CAP);  // [MAXSEG * CAP]
  const DivU32 dper = make_divu32(static_cast<uint32_t>(pad.per));
  auto pw = [&](uint32_t w) -> int {  // padded index of segment word w
    const uint32_t q = divu32(dper, w);
    return static_cast<int>(q * pad.stride + (w - q * pad.per));
  };
  int n = static_cast<int>(a.n_cols);
  if (a.valid_len) {
    const int64_t v = __ldg(a.valid_len + r);
    n = v < 0 ? 0 : (v < n ? static_cast<int>(v) : n);
  }
  const int s0 = s * static_cast<int>(seg_len);
  const int s1 = s0 + static_cast<int>(seg_len) < static_cast<int>(a.n_cols) ? s0 + static_cast<int>(seg_len)
                                                                              : static_cast<int>(a.n_cols);
  const int nw_seg = s1 > s0 ? (s1 - s0 + 31) / 32 : 0;
  const float* row = a.scores + static_cast<int64_t>(r) * a.ld;
  const int lim = ((n + 3) & ~3) < a.ld ? ((n + 3) & ~3) : static_cast<int>(a.ld);
  for (int i = t; i < bm_words; i += NT) tb[i] = 0;
  // The row's histogram and the segment's scores (up to the row's length
  // rounded to 16 bytes) come into shared memory by 16-byte cp.async copies of
  // every thread, consecutive threads on consecutive bytes: one commit group
  // for the histogram and one per collect round, each round's copies issued
  // kAhead rounds before it is processed.  (Issuing every round at once made
  // the first round's processing slow, its shared-memory reads meeting the
  // later rounds' copies as they landed, and the issue itself stall on the
  // copies in flight; large bulk copies delivered far fewer bytes per
  // microsecond.)
  constexpr int kAhead = 2;
  const int s1r = (s1 + 3) & ~3;  // whole 16-byte groups
  const int s_hi = s1r < lim ? s1r : lim;
  const int n_rounds = s1 > s0 ? (s1 - s0 + kColRound - 1) / kColRound : 0;
  bool staged_ok = true;
  const bool staging = live;
  auto issue_round = [&](int i) {
#pragma unroll
    for (int k = 0; k < kColRound / 4 / NT; ++k) {
      const int p = s0 + i * kColRound + 4 * (k * NT + t);
      // groups past the staged range are zero-filled (read nothing)
      tc::cp_async16_zfill(seg + (p - s0), row + (p < s_hi ? p : s0), p < s_hi ? 16u : 0u);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  const int first_rounds = n_rounds < kAhead ? n_rounds : kAhead;
  if (staging) {
    const uint32_t* hsrc = L.hist + static_cast<int64_t>(r) * kB1;
#pragma unroll
    for (int k = 0; k < kB1 / 4 / NT; ++k)
      tc::cp_async16_zfill(hsm + 4 * (k * NT + t), hsrc + 4 * (k * NT + t), 16u);
    asm volatile("cp.async.commit_group;" ::: "memory");
    for (int i = 0; i < first_rounds; ++i) issue_round(i);
  }
  // waits until at most `pending` of this thread's newest groups are in flight
  auto wait_groups = [&](int pending) {
    switch (pending) {
      case 0: asm volatile("cp.async.wait_group 0;" ::: "memory"); break;
      case 1: asm volatile("cp.async.wait_group 1;" ::: "memory"); break;
      case 2: asm volatile("cp.async.wait_group 2;" ::: "memory"); break;
      case 3: asm volatile("cp.async.wait_group 3;" ::: "memory"); break;
      default: asm volatile("cp.async.wait_group 4;" ::: "memory"); break;
    }
  };
  if (staging) {
    wait_groups(first_rounds);  // the histogram
    tk_sync<NT, ID>();          // every thread's part of it
  }
  // ---------------------------------------------------------------- collect
  uint32_t keff = 0, b1 = 0xffffffffu, rank1 = 0;
  int nc = 0, above = 0;
  if (live && staged_ok) {
    uint32_t hv[kB1 / NT];
#pragma unroll
    for (int i = 0; i < kB1 / NT; ++i) hv[i] = hsm[t * (kB1 / NT) + i];
    const uint32_t total = tk_find<NT, ID, kB1>(hv, static_cast<uint32_t>(a.k), S, true);
    keff = total < static_cast<uint32_t>(a.k) ? total : static_cast<uint32_t>(a.k);
    if (keff > 0) {
      b1 = static_cast<uint32_t>(S.s_bin);
      rank1 = S.s_rank;
    }
#pragma unroll 1
    for (int rd = 0; keff > 0 && rd < n_rounds; ++rd) {
      // round rd + kAhead's copies go out; this round's have had kAhead rounds to land
      if (rd + kAhead < n_rounds) issue_round(rd + kAhead);
      const int later = n_rounds - 1 - rd;  // rounds after this one, issued by now
      wait_groups(later < kAhead ? later : kAhead);
      tk_sync<NT, ID>();  // every thread's part of them
      // thread t builds bitmap word t of the round (positions 32 t .. 32 t + 31)
      // from its own 16-byte groups, read in a rotated order so that the
      // warp's reads spread over the banks; every bit is independent work
      const int base = s0 + rd * kColRound;
      const int q = base + 32 * t;
      const float4* g4 = reinterpret_cast<const float4*>(seg + (q - s0));
      uint32_t above_w = 0u, bin_w = 0u;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const int vv = (v + lane) & 7;
        const int p = q + 4 * vv;
        const float4 x = p < s_hi ? g4[vv] : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        const float xs[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t k = p + e < n ? order_key(xs[e]) : 0u;
          const uint32_t hi = k >> 20;
          above_w |= static_cast<uint32_t>(k != 0u && hi > b1) << (4 * vv + e);
          bin_w |= static_cast<uint32_t>(k != 0u && hi == b1) << (4 * vv + e);
        }
      }
      const int wi = rd * (kColRound / kWordElems) + t;
      if (wi < nw_seg) bm[pw(static_cast<uint32_t>(wi))] = above_w;
      above += __popc(above_w);
      const int ncl = __popc(bin_w);
      int tot;
      const int off = tk_excl_scan<NT, ID>(ncl, S.warp_sums, &tot);
      int o = nc + off;
      while (bin_w) {  // this thread's candidates, in position order
        const int b = __ffs(bin_w) - 1;
        bin_w &= bin_w - 1;
        if (o < CAP) cs[o] = make_uint2(order_key(seg[q - s0 + b]), static_cast<uint32_t>(q + b));
        ++o;
      }
      nc += tot;
    }
  }
  if (!staged_ok) live = false;
  // words of the bitmap the rounds did not write (a segment without a selectable key)
  if (!live || keff == 0)
    for (int i = t; i < bm_words; i += NT) bm[i] = 0;
  if (t == 0) hdr->nc = static_cast<uint32_t>(nc);
  tc::cluster_sync();  // ---- every segment collected
  // ---------------------------------------------------------------- threshold key T
  // every CTA's candidate count and keys, copied into this CTA's shared
  // memory with all of the remote loads in flight at once (a remote load is a
  // round trip; one after another they would cost a round trip each)
  const uint32_t hdr_u = tc::smem_u32(hdr), cs_u = tc::smem_u32(cs);
  uint32_t ncq[MAXSEG];
#pragma unroll
  for (int q = 0; q < MAXSEG; ++q)
    ncq[q] = q < ns ? tc::ld_cluster_u32(tc::cluster_map(hdr_u, static_cast<uint32_t>(q))) : 0u;
  bool ovf = false;
  int n_all = 0;
  uint32_t offq[MAXSEG];
#pragma unroll
  for (int q = 0; q < MAXSEG; ++q) {
    ovf |= ncq[q] > static_cast<uint32_t>(CAP);
    offq[q] = static_cast<uint32_t>(n_all);
    n_all += static_cast<int>(ncq[q]);
  }
  if (live && keff > 0 && !ovf) {
    constexpr int U = CAP / NT;
    uint32_t kv[MAXSEG][U];
#pragma unroll
    for (int q = 0; q < MAXSEG; ++q) {
      const uint32_t base_q = tc::cluster_map(cs_u, static_cast<uint32_t>(q < ns ? q : 0));
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t c = static_cast<uint32_t>(t + u * NT);
        kv[q][u] = c < ncq[q] ? tc::ld_cluster_u32(base_q + c * 8u) : 0u;
      }
    }
#pragma unroll
    for (int q = 0; q < MAXSEG; ++q) {
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const uint32_t c = static_cast<uint32_t>(t + u * NT);
        if (c < ncq[q]) allk[offq[q] + c] = kv[q][u];
      }
    }
  }
  uint32_t T = 0, ties = 0;
  const bool work = live && keff > 0;
  if (ovf) {
    // Some CTA's list overflowed (many keys in the threshold bin, e.g. a
    // large k or a flat score distribution).  T's lower two digits are then
    // counted from every CTA's own segment, still in its shared memory, and
    // the counts summed across the cluster through distributed shared memory:
    // two rounds of two cluster barriers, every CTA taking part (the barriers
    // are the cluster's, live or not).
    T = b1 << 20;
    uint32_t rank = rank1;
    constexpr int PER = 1024 / NT;
    static_assert(PER == 4, "one 16-byte word of bins per thread");
    for (int pass = 0; pass < 2; ++pass) {
      const uint32_t shift = pass == 0 ? 10 : 0;
      const uint32_t pre_shift = pass == 0 ? 20 : 10;
      const uint32_t prefix = T >> pre_shift;
      for (int i = t; i < 1024; i += NT) S.h[i] = 0;
      tk_sync<NT, ID>();
      if (work) {
        for (int p = s0 + t; p < s1 && p < n; p += NT) {
          const uint32_t key = order_key(seg[p - s0]);
          if (key != 0u && (key >> pre_shift) == prefix) atomicAdd(&S.h[(key >> shift) & 1023u], 1u);
        }
      }
      tc::cluster_sync();  // every CTA's counts are complete
      if (work) {
        // bins 4t .. 4t+3 of every CTA, all loads in flight, then summed
        const uint32_t h_u = tc::smem_u32(&S.h[t * PER]);
        float4 part[MAXSEG];
#pragma unroll
        for (int q = 0; q < MAXSEG; ++q)
          part[q] = q < ns ? tc::ld_cluster_f4(tc::cluster_map(h_u, static_cast<uint32_t>(q)))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        uint32_t hl[PER] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int q = 0; q < MAXSEG; ++q) {
          hl[0] += __float_as_uint(part[q].x);
          hl[1] += __float_as_uint(part[q].y);
          hl[2] += __float_as_uint(part[q].z);
          hl[3] += __float_as_uint(part[q].w);
        }
        tk_find<NT, ID, 1024>(hl, rank, S, false);
        T |= static_cast<uint32_t>(S.s_bin) << shift;
        rank = S.s_rank;
      }
      tc::cluster_sync();  // every CTA has read the others' counts before they are cleared
    }
    ties = rank;
  } else if (work) {
    {
      for (int pass = 0; pass < 2; ++pass) {
        for (int i = t; i < 1024; i += NT) S.h[i] = 0;
        tk_sync<NT, ID>();  // also: the gathered keys are complete
        const uint32_t shift = pass == 0 ? 10 : 0;
        const uint32_t pre_shift = pass == 0 ? 20 : 10;
        const uint32_t prefix = pass == 0 ? b1 : (T >> 10);
        for (int c = t; c < n_all; c += NT) {
          const uint32_t key = allk[c];
          if ((key >> pre_shift) == prefix) atomicAdd(&S.h[(key >> shift) & 1023u], 1u);
        }
        tk_sync<NT, ID>();
        uint32_t hl[1024 / NT];
#pragma unroll
        for (int i = 0; i < 1024 / NT; ++i) hl[i] = S.h[t * (1024 / NT) + i];
        tk_find<NT, ID, 1024>(hl, pass == 0 ? rank1 : ties, S, false);
        const uint32_t bb = static_cast<uint32_t>(S.s_bin);
        T = pass == 0 ? ((b1 << 20) | (bb << 10)) : (T | bb);
        ties = S.s_rank;
        tk_sync<NT, ID>();
      }
    }
  }
  if (work) {
    // this segment's keys of bin b1: above T into the bitmap, equal to T into the tie bitmap
    if (!ovf) {
      for (int c = t; c < nc; c += NT) {
        const uint2 e = cs[c];
        const uint32_t w = (e.y - static_cast<uint32_t>(s0)) >> 5;
        if (e.x > T) atomicOr(&bm[pw(w)], 1u << (e.y & 31));
        else if (e.x == T) atomicOr(&tb[pw(w)], 1u << (e.y & 31));
      }
    } else {
      for (int p = s0 + t; p < s1 && p < n; p += NT) {
        const uint32_t key = order_key(seg[p - s0]);
        if ((key >> 20) != b1) continue;
        const uint32_t w = static_cast<uint32_t>(p - s0) >> 5;
        if (key > T) atomicOr(&bm[pw(w)], 1u << (p & 31));
        else if (key == T) atomicOr(&tb[pw(w)], 1u << (p & 31));
      }
    }
  }
  tk_sync<NT, ID>();
  // ---------------------------------------------------------------- counts
  const int w0 = t * pad.per;
  const int nmine = nw_seg - w0 < pad.per ? (nw_seg - w0 > 0 ? nw_seg - w0 : 0) : pad.per;
  const int pb = t * pad.stride;
  int my_gt = 0, my_eq = 0;
  for (int i = 0; i < nmine; ++i) {
    my_gt += __popc(bm[pb + i]);
    my_eq += __popc(tb[pb + i]);
  }
  int gt_tot, eq_tot;
  tk_excl_scan<NT, ID>(my_gt, S.warp_sums, &gt_tot);
  int eq_before = tk_excl_scan<NT, ID>(my_eq, S.warp_sums, &eq_tot);
  if (t == 0) {
    hdr->gt = static_cast<uint32_t>(gt_tot);
    hdr->eq = static_cast<uint32_t>(eq_tot);
  }
  tc::cluster_sync();  // ---- every segment's counts published
  // entries before this segment and the ties left to it (lowest positions
  // first); the remote counts are loaded together
  uint32_t gtq[MAXSEG], eqq[MAXSEG];
#pragma unroll
  for (int q = 0; q < MAXSEG; ++q) {
    gtq[q] = q < ns ? tc::ld_cluster_u32(tc::cluster_map(hdr_u + 4u, static_cast<uint32_t>(q))) : 0u;
    eqq[q] = q < ns ? tc::ld_cluster_u32(tc::cluster_map(hdr_u + 8u, static_cast<uint32_t>(q))) : 0u;
  }
  uint32_t off = 0, ties_mine = 0, eq_seen = 0;
#pragma unroll
  for (int q = 0; q < MAXSEG; ++q) {
    const uint32_t gt_q = gtq[q], eq_q = eqq[q];
    const uint32_t left = ties > eq_seen ? ties - eq_seen : 0u;
    const uint32_t take = left < eq_q ? left : eq_q;
    if (q < s) off += gt_q + take;
    if (q == s) ties_mine = take;
    eq_seen += eq_q;
  }
  // no CTA reads another's shared memory past this point: the arrival lets
  // the others leave once they are done; this CTA waits before it leaves
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
  // ---------------------------------------------------------------- compaction
  int32_t* out = a.idx + static_cast<int64_t>(r) * a.k;
  if (live) {
    int my_sel = 0;
    for (int i = 0; i < nmine; ++i) {
      const uint32_t x = tb[pb + i];
      const int px = __popc(x);
      const int take = static_cast<int>(ties_mine) - eq_before;
      uint32_t add = 0;
      if (take > 0) add = take >= px ? x : low_bits(x, take);
      eq_before += px;
      const uint32_t merged = bm[pb + i] | add;
      bm[pb + i] = merged;
      my_sel += __popc(merged);
    }
    int sel_tot;
    int o = static_cast<int>(off) + tk_excl_scan<NT, ID>(my_sel, S.warp_sums, &sel_tot);
    for (int i = 0; i < nmine; ++i) {
      uint32_t x = bm[pb + i];
      while (x) {
        const int b = __ffs(x) - 1;
        x &= x - 1;
        if (o < a.k) out[o] = s0 + (w0 + i) * 32 + b;
        else record_error(a.status, LSA_ERR_BOUNDS, r, o);  // cannot happen if the counts agree
        ++o;
      }
    }
    for (int i = static_cast<int>(keff) + s * NT + t; i < a.k; i += ns * NT) out[i] = -1;
    if (a.wait_ctr) {
      // decode step: the last CTA of the row to finish raises the row's flag
      // (the attention of row r may read its selection from then on).  The
      // barrier orders this CTA's output writes before thread 0's release;
      // the last adder has acquired the others' and releases all of them.
      tk_sync<NT, ID>();
      if (t == 0) {
        const uint32_t done = tc::atom_acq_rel_gpu_add(L.row_done + r, 1u);
        if (done == static_cast<uint32_t>(ns - 1)) tc::st_release_gpu(L.sel_done + r, 1u);
      }
    }
  }
  tc::cluster_wait();  // ---- the others have read this CTA's shared memory
  if (staging) asm volatile("cp.async.wait_all;" ::: "memory");  // nothing in flight when the CTA leaves
}

}  // namespace tk
}  // namespace lsa
