"""CPU oracle for one DeepSeek-Sparse-Attention (DSA) decode step.

TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it, and it shares no code,
table or helper with that path.

It is a plain, slow, fp64 restatement of what the step computes:

  1. Lightning-indexer scan.  Before each DSA layer the lightning indexer scores
     every cached token of the sequence and the layer attends only the k = 2048
     best (MLI "Multi-layer Indexer" abstract, zhuanzhiai.com, sentence 2).  The
     score of token s for a query row is DSA's lightning-indexer form
         I(s) = sum_h  w_h * ReLU(q_h . k_s)
     (DeepSeek-V3.2-Exp technical report, the DSA source listed on the
     LeanSparse episode page).  FP8 keys carry a per-token scale:
     k_s = scale_s * e4m3(k_s).
  2. Top-k.  Keep the k tokens with the largest scores; equal scores go to the lower
     position; -inf (masked) and NaN are never kept; the kept positions are
     returned sorted ascending and padded with -1.
  3. Sparse attention over the kept rows only (the LeanSparse episode page's
     point that sparse attention cuts what is read, not what is stored): softmax(scale * q . K_sel)
     weighted sum of V_sel, V being the first v_dim columns of the KV row, plus
     the log-sum-exp of the scaled logits.
  Prefill variant: a chunk of query rows at positions p_i scores the cache
  under a causal mask (position s is visible iff s <= p_i); the rest of the
  step is unchanged per row.

Every function below is written from those definitions; no blocking, fusion or
reordering beyond them.  Inputs are the stored bits (bf16 as uint16, e4m3fn as
uint8), decoded exactly to fp64 here.
"""
from __future__ import annotations

import numpy as np

# ---------------------------------------------------------------------------
# 1. exact decoding of the stored element formats


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 is the upper half of an IEEE binary32: value = float32(bits << 16)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def e4m3_to_f64(bits: np.ndarray) -> np.ndarray:
    """OCP FP8 E4M3 ('fn' variant): 1 sign, 4 exponent (bias 7), 3 mantissa bits.

    exponent field 0 -> subnormal m/8 * 2^-6; S.1111.111 -> NaN; no infinities.
    """
    b = np.asarray(bits, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    sub = (m / 8.0) * 2.0 ** -6
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & (m == 7), np.nan, val)


def decode(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "bf16":
        return bf16_to_f64(x)
    if dtype == "fp8":
        return e4m3_to_f64(x)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# cache addressing: logical position -> stored row


def physical_rows(b: int, positions: np.ndarray, block_table, block_size: int, stride: int) -> np.ndarray:
    """Flat row numbers of logical positions of sequence b.

    Paged: row = block_table[b][pos // bs] * bs + pos % bs.  Contiguous: b * stride + pos.
    """
    pos = np.asarray(positions, dtype=np.int64)
    if block_size > 0:
        blk = np.asarray(block_table)[b, pos // block_size].astype(np.int64)
        assert (blk >= 0).all(), "block table entry missing for a visible position"
        return blk * block_size + pos % block_size
    return b * stride + pos


def cache_rows(storage: np.ndarray, b: int, positions, block_table, block_size: int, stride: int) -> np.ndarray:
    flat = storage.reshape(-1, *storage.shape[2:]) if storage.ndim >= 3 else storage.reshape(-1)
    return flat[physical_rows(b, positions, block_table, block_size, stride)]


# ---------------------------------------------------------------------------
# 2. lightning-indexer scores


def indexer_scores(q_idx: np.ndarray, w: np.ndarray, keys: np.ndarray, scales=None, pos=None) -> np.ndarray:
    """I(s) = sum_h w[h] * max(0, scale_s * sum_d q_idx[h, d] * keys[s, d]).

    q_idx [H_I, d_I], w [H_I], keys [L, d_I] (fp64); scales [L] or None.
    With pos given (causal prefill), positions s > pos are -inf.
    """
    q_idx = np.asarray(q_idx, np.float64)
    keys = np.asarray(keys, np.float64)
    dots = keys @ q_idx.T                      # [L, H_I]: q_h . k_s
    if scales is not None:
        dots = dots * np.asarray(scales, np.float64)[:, None]
    scores = np.maximum(dots, 0.0) @ np.asarray(w, np.float64)
    if pos is not None:
        scores[int(pos) + 1:] = -np.inf
    return scores


# ---------------------------------------------------------------------------
# 3. top-k with lowest-position tie-break


def topk(scores: np.ndarray, valid_len: int, k: int) -> np.ndarray:
    """Positions of the min(k, #selectable) largest entries of scores[:valid_len].

    Order: score descending, then position ascending (equal scores -> the lower
    position wins; -0.0 equals +0.0).  -inf and NaN are not selectable.  The
    result is sorted ascending and padded with -1 to length k.  Comparisons are
    made in the dtype of ``scores`` (fp32 scores compare as fp32).
    """
    s = np.asarray(scores)[:int(valid_len)]
    pos = np.arange(s.shape[0])
    ok = ~(np.isnan(s) | (s == -np.inf))
    s_ok, pos_ok = s[ok], pos[ok]
    order = np.lexsort((pos_ok, -s_ok))       # last key is primary
    take = np.sort(pos_ok[order[:k]])
    out = np.full(k, -1, np.int32)
    out[:take.shape[0]] = take
    return out


# ---------------------------------------------------------------------------
# 4. attention over a given list of rows


def attention(q: np.ndarray, kv_rows: np.ndarray, v_dim: int, scale: float):
    """Softmax attention of each head over the given KV rows (fp64).

    q [H, D]; kv_rows [n, D]; logits z = scale * q . kv_row; V = kv_rows[:, :v_dim].
    Returns o [H, v_dim] and lse [H] = log sum_j exp(z_j).  n == 0 gives o = 0,
    lse = -inf.
    """
    q = np.asarray(q, np.float64)
    kv = np.asarray(kv_rows, np.float64)
    H = q.shape[0]
    if kv.shape[0] == 0:
        return np.zeros((H, v_dim)), np.full(H, -np.inf)
    z = scale * (q @ kv.T)                     # [H, n]
    m = z.max(axis=1, keepdims=True)
    e = np.exp(z - m)
    l = e.sum(axis=1, keepdims=True)
    p = e / l
    o = p @ kv[:, :v_dim]
    lse = (m + np.log(l))[:, 0]
    return o, lse


def sparse_attention(q: np.ndarray, kv_storage, b: int, idx: np.ndarray, block_table, block_size: int,
                     stride: int, kv_dtype: str, v_dim: int, scale: float):
    """Attention of one query row over the KV rows at positions idx (-1 entries skipped)."""
    sel = np.asarray(idx)
    sel = sel[sel >= 0]
    rows = decode(cache_rows(kv_storage, b, sel, block_table, block_size, stride), kv_dtype)
    return attention(q, rows, v_dim, scale)


# ---------------------------------------------------------------------------
# whole-row helpers on a synthetic case


def row_visible(case, r: int) -> int:
    b = int(case.row_seq[r])
    L = int(case.seq_lens[b])
    if case.row_pos is not None:
        return min(L, int(case.row_pos[r]) + 1)
    return L


def row_scores(case, r: int) -> np.ndarray:
    """Scores of query row r over positions [0, seq_len) of its sequence (fp64)."""
    s = case.spec
    b = int(case.row_seq[r])
    L = int(case.seq_lens[b])
    pos = np.arange(L)
    keys = decode(cache_rows(case.idx_keys, b, pos, case.block_table, s.block_size, s.stride), s.idx_key_dtype)
    scales = None
    if case.idx_scales is not None:
        scales = cache_rows(case.idx_scales, b, pos, case.block_table, s.block_size, s.stride).astype(np.float64)
    qi = decode(case.q_idx[r], s.act_dtype)
    p = None if case.row_pos is None else int(case.row_pos[r])
    return indexer_scores(qi, case.w[r].astype(np.float64), keys, scales, p)


def row_step(case, r: int, k: int = None):
    """Full step for query row r: (scores fp64, selection, o, lse)."""
    s = case.spec
    k = s.top_k if k is None else k
    sc = row_scores(case, r)
    sel = topk(sc, sc.shape[0], k)
    o, lse = sparse_attention(decode(case.q[r], s.act_dtype), case.kv, int(case.row_seq[r]), sel,
                              case.block_table, s.block_size, s.stride, s.act_dtype, s.v_dim,
                              s.softmax_scale)
    return sc, sel, o, lse


def row_attention(case, r: int, idx: np.ndarray):
    s = case.spec
    return sparse_attention(decode(case.q[r], s.act_dtype), case.kv, int(case.row_seq[r]), idx,
                            case.block_table, s.block_size, s.stride, s.act_dtype, s.v_dim,
                            s.softmax_scale)


def decode_step(case, rows=None, threads: int = 1):
    """Run row_step over the given rows (default all).  Returns lists per row."""
    rows = list(range(case.rows)) if rows is None else list(rows)
    if threads > 1:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(threads) as ex:
            res = list(ex.map(lambda r: row_step(case, r), rows))
    else:
        res = [row_step(case, r) for r in rows]
    return rows, res


# --------------------------------------------------------------------------- several layers
# A decode step runs one DSA layer after another.  The MLI page ("Multi-layer
# Indexer" abstract, zhuanzhiai.com) fixes two routings of the selections:
#  - IndexCache (sentences 8-9): only a fraction 1/r of the layers (the
#    retention) keep an indexer; a layer without one reuses the selection of
#    the latest layer that has one.  With r = 1 every layer attends its own
#    selection: plain DSA.
#  - MLI (sentences 4-5): a layer attends the selection of the previous indexer
#    layer instead of its own, so its indexer no longer gates its attention.
# Readings where the page is silent: the layers that keep an indexer are 0, r,
# 2r, ...; layer 0 has no earlier indexer layer and attends its own selection.

ROUTE_OWN = 0   # IndexCache (DSA at r = 1): the latest indexer layer i <= l
ROUTE_PREV = 1  # MLI: the latest indexer layer i < l (layer 0: its own)


def indexer_layers(n_layers: int, retention: int) -> list:
    """Layers that keep an indexer at retention 1/retention."""
    return [l for l in range(n_layers) if l % retention == 0]


def selection_source(n_layers: int, retention: int, route: int) -> list:
    """For every layer, the layer whose indexer selection it attends."""
    keep = indexer_layers(n_layers, retention)
    src = []
    for l in range(n_layers):
        before = [i for i in keep if (i <= l if route == ROUTE_OWN else i < l)]
        src.append(before[-1] if before else 0)
    return src


def decode_layers(layers, retention: int, route: int):
    """Several layers of one decode batch (a list of cases sharing the
    sequence lengths and block table).  Each layer attends, with its own query
    and KV cache, the selection its route names; an indexer layer's selection
    is the top-k of its own scores.  Returns the source table and per layer
    (selection attended [rows, k], o [rows, H, D_v], lse [rows, H])."""
    src = selection_source(len(layers), retention, route)
    sel = {}
    for i in sorted(set(src)):
        c = layers[i]
        sel[i] = np.stack([topk(row_scores(c, r), row_visible(c, r), c.spec.top_k) for r in range(c.rows)])
    res = []
    for l, c in enumerate(layers):
        idx = sel[src[l]]
        att = [row_attention(c, r, idx[r]) for r in range(c.rows)]
        res.append((idx, np.stack([a[0] for a in att]), np.stack([a[1] for a in att])))
    return src, res


# --------------------------------------------------------------------------- two-stage indexer
# The LeanSparse episode page (summary paragraph) proposes, for decode, to
# search compact indexer keys and fetch only a short list of the original keys
# to rank exactly.  Readings where the page is silent: the compact keys are
# e4m3 with one fp32 scale per token (the FP8 indexer-key form); the short
# list is the n_cand best tokens by their compact scores (ties to the lower
# position, as the top-k); the exact ranking is the top-k of those candidates
# by their scores with the original keys.

def compact_row_scores(case, compact_bits: np.ndarray, compact_scales: np.ndarray, r: int) -> np.ndarray:
    """Scores of row r over its sequence with the compact keys (fp64)."""
    s = case.spec
    b = int(case.row_seq[r])
    L = int(case.seq_lens[b])
    pos = np.arange(L)
    keys = e4m3_to_f64(cache_rows(compact_bits, b, pos, case.block_table, s.block_size, s.stride))
    scales = cache_rows(compact_scales, b, pos, case.block_table, s.block_size, s.stride).astype(np.float64)
    qi = decode(case.q_idx[r], s.act_dtype)
    return indexer_scores(qi, case.w[r].astype(np.float64), keys, scales, None)


def two_stage_select(case, compact_bits: np.ndarray, compact_scales: np.ndarray, r: int, k: int,
                     n_cand: int) -> np.ndarray:
    """Row r's selection by the two-stage search: the n_cand candidates of the
    compact scores, ranked by their exact scores (the case's own keys); k
    positions sorted ascending, -1 padded."""
    L = row_visible(case, r)
    cand = topk(compact_row_scores(case, compact_bits, compact_scales, r), L, n_cand)
    cand = cand[cand >= 0]
    exact = np.full(L, -np.inf)
    exact[cand] = row_scores(case, r)[cand]
    return topk(exact, L, k)


# --------------------------------------------------------------------------- block selection
# The SparDA abstract (page 4 of the sources) has the selector pick the KV
# *blocks* a layer needs, and a forecast of the next layer's blocks lets their
# host-to-device copy run while the current layer computes.  Readings where
# the page is silent: a block is one cache page (block_size consecutive
# positions); a block's score is the largest indexer score of its visible
# tokens (the trained Forecast projection is out of scope, so the indexer's
# own token scores stand in for the selector's); the kept blocks are the
# n_blocks best by block score with ties to the lower block, ascending, -1
# padded; the layer then attends every visible token of its kept blocks.

def block_scores(scores: np.ndarray, valid_len: int, block_size: int) -> np.ndarray:
    """Per block of block_size positions: the largest score among its positions
    below valid_len (-inf for a block with none, NaN ignored)."""
    s = np.asarray(scores, np.float64)[:int(valid_len)]
    nb = (s.shape[0] + block_size - 1) // block_size
    out = np.full(nb, -np.inf)
    for blk in range(nb):
        vals = s[blk * block_size:(blk + 1) * block_size]
        vals = vals[~np.isnan(vals)]
        if vals.size:
            out[blk] = vals.max()
    return out


def block_select(scores: np.ndarray, valid_len: int, block_size: int, n_blocks: int) -> np.ndarray:
    """The n_blocks best blocks by block score (ties to the lower block),
    ascending, padded with -1."""
    bs = block_scores(scores, valid_len, block_size)
    return topk(bs, bs.shape[0], n_blocks)


def block_positions(blocks: np.ndarray, block_size: int, valid_len: int) -> np.ndarray:
    """Every position below valid_len inside the given blocks (-1 skipped), ascending."""
    pos = [b * block_size + t for b in np.asarray(blocks) if b >= 0 for t in range(block_size)
           if b * block_size + t < valid_len]
    return np.array(sorted(pos), np.int64)


def row_block_step(case, r: int, n_blocks: int, q_row=None, block_size: int = None):
    """Row r of a case: its kept blocks of block_size positions (default the
    cache's page size) by its indexer scores, the positions they cover, and the
    attention of q_row (default the row's own attention query, decoded) over
    those positions."""
    s = case.spec
    bs = s.block_size if block_size is None else block_size
    L = row_visible(case, r)
    blocks = block_select(row_scores(case, r), L, bs, n_blocks)
    pos = block_positions(blocks, bs, L)
    q = decode(case.q[r], s.act_dtype) if q_row is None else q_row
    o, lse = sparse_attention(q, case.kv, int(case.row_seq[r]), pos, case.block_table, s.block_size, s.stride,
                              s.act_dtype, s.v_dim, s.softmax_scale)
    return blocks, pos, o, lse
