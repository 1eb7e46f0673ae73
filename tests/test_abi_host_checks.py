"""Host-side argument checks of every C-ABI entry point.

The boundary's contract (include/lsa.h, "Conventions"): an argument error the
host can see returns its code and enqueues nothing, and a call with nothing to
do returns LSA_OK without touching the device.  Both paths end before any CUDA
call, so these tests run without a GPU; the pointers are fake, aligned device
addresses that the library never dereferences on these paths.
"""
import ctypes

import pytest

from sparse_attention_decode_scan_b200 import lsa, synth
from sparse_attention_decode_scan_b200.device import make_dims

OK, INVALID, UNSUPPORTED, WORKSPACE = lsa.LSA_OK, lsa.LSA_ERR_INVALID_ARG, lsa.LSA_ERR_UNSUPPORTED, lsa.LSA_ERR_WORKSPACE
A = 0x10000000            # an aligned fake device address
MISALIGNED = A + 8        # 8-byte aligned, not 16
WS = ctypes.c_void_p(0x20000000)
BIG = 1 << 40             # workspace bytes that satisfy every size check


@pytest.fixture(scope="module", autouse=True)
def built():
    from sparse_attention_decode_scan_b200 import build
    build.build()


def _dims(name=synth.DECODE_B32, **kw):
    d = make_dims(synth.WORKLOADS[name])
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def _cache(d, batch=4, max_len=4096, **kw):
    c = lsa.Cache()
    c.idx_keys, c.idx_key_scales, c.kv = A, (A if d.idx_key_dtype == lsa.LSA_FP8_E4M3 else None), A
    paged = d.block_size > 0
    c.block_table = A if paged else None
    c.max_blocks_per_seq = (max_len + d.block_size - 1) // d.block_size if paged else 0
    c.n_blocks = max(batch, 1) * c.max_blocks_per_seq if paged else 0
    c.max_len, c.seq_lens, c.batch = max_len, A, batch
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _scores(d, c, rows=4, row_seq=None, row_pos=None, q_idx=A, w=A, scores=A, ld=None, ws=WS, ws_bytes=BIG):
    ld = c.max_len if ld is None else ld
    return lsa.lib().lsa_indexer_scores(ctypes.byref(d), ctypes.byref(c), rows, row_seq, row_pos, q_idx, w, scores,
                                        ld, ws, ws_bytes, None)


def test_indexer_scores_checks():
    d = _dims()
    c = _cache(d)
    assert _scores(d, c, rows=0) == OK                           # nothing to do
    assert _scores(_dims(n_idx_heads=0), c) == INVALID
    assert _scores(_dims(idx_dim=12), c) == INVALID               # not a multiple of 8
    assert _scores(d, c, rows=-1) == INVALID
    assert _scores(d, c, ld=c.max_len - 4) == INVALID            # ld below max_len
    assert _scores(d, c, q_idx=MISALIGNED) == INVALID
    assert _scores(d, c, w=None) == INVALID
    assert _scores(d, c, rows=5) == INVALID                      # more rows than sequences, no row map
    assert _scores(d, c, rows=70000, row_seq=A) == UNSUPPORTED
    assert _scores(d, _cache(d, block_table=None)) == INVALID    # paged without a block table
    assert _scores(d, _cache(d, max_blocks_per_seq=1)) == INVALID  # pages cannot hold max_len
    fp8 = _dims(synth.DECODE_B4_FP8)
    assert _scores(fp8, _cache(fp8, idx_key_scales=None)) == INVALID  # FP8 keys need their scales
    assert _scores(d, c, ws=None) == WORKSPACE
    assert _scores(d, c, ws=ctypes.c_void_p(0x20000010)) == WORKSPACE  # not 256-byte aligned
    assert _scores(d, c, ws_bytes=16) == WORKSPACE


def _topk(rows=4, ld=4096, n_cols=4096, k=2048, scores=A, idx=A, ws=WS, ws_bytes=BIG):
    return lsa.lib().lsa_topk(scores, ld, rows, A, n_cols, k, idx, ws, ws_bytes, None)


def test_topk_checks():
    assert _topk(rows=0) == OK
    assert _topk(k=0) == INVALID
    assert _topk(ld=4094, n_cols=4094) == INVALID                 # ld not a multiple of 4
    assert _topk(ld=4092) == INVALID                              # ld below n_cols
    assert _topk(scores=MISALIGNED) == INVALID
    assert _topk(idx=None) == INVALID
    assert _topk(rows=70000) == UNSUPPORTED
    assert _topk(ld=1 << 31, n_cols=1 << 31) == UNSUPPORTED       # positions beyond int32
    assert _topk(ws_bytes=16) == WORKSPACE
    noalloc = lsa.lib().lsa_topk_noalloc
    assert noalloc(A, 4096, 4, A, 4096, 0, A, None) == INVALID
    assert noalloc(A, 4096, 70000, A, 4096, 2048, A, None) == UNSUPPORTED


def _attn(d, c, rows=4, row_seq=None, q=A, idx=A, out=A, ws=WS, ws_bytes=BIG):
    return lsa.lib().lsa_sparse_attn_decode(ctypes.byref(d), ctypes.byref(c), rows, row_seq, q, idx, out, None, ws,
                                            ws_bytes, None)


def test_sparse_attn_checks():
    d = _dims()
    c = _cache(d)
    assert _attn(d, c, rows=0) == OK
    assert _attn(_dims(v_dim=1024), c) == INVALID                 # v_dim above qk_dim
    assert _attn(d, _cache(d, kv=None)) == INVALID
    assert _attn(d, c, q=MISALIGNED) == INVALID
    assert _attn(d, c, out=MISALIGNED) == INVALID
    assert _attn(d, c, rows=5) == INVALID
    assert _attn(d, c, rows=70000, row_seq=A) == UNSUPPORTED
    assert _attn(d, c, ws_bytes=16) == WORKSPACE


def _step(d, c, flags=0, q_idx=A, q=A, out=A, ws=WS, ws_bytes=BIG):
    return lsa.lib().lsa_decode_step(ctypes.byref(d), ctypes.byref(c), q_idx, A, q, out, None, None, flags, ws,
                                     ws_bytes, None)


def test_decode_step_checks():
    d = _dims()
    assert _step(d, _cache(d, batch=0)) == OK                     # no sequence: nothing to do
    c = _cache(d)
    assert _step(d, c, flags=7) == INVALID
    assert _step(d, c, q_idx=MISALIGNED) == INVALID
    assert _step(d, c, q=None) == INVALID
    assert _step(d, _cache(d, idx_keys=None)) == INVALID          # the step needs the indexer keys
    assert _step(d, _cache(d, batch=70000)) == UNSUPPORTED
    assert _step(d, c, ws_bytes=16) == WORKSPACE
    ev = (ctypes.c_void_p * 4)()
    assert lsa.lib().lsa_decode_step_profiled(ctypes.byref(d), ctypes.byref(c), A, A, A, A, None, None, 3, WS, BIG,
                                              None, ev) == INVALID


def test_candidate_and_two_stage_checks():
    d = _dims()
    c = _cache(d)
    cand = lsa.lib().lsa_candidate_scores
    assert cand(ctypes.byref(d), ctypes.byref(c), 0, None, None, A, A, A, 8, A, 8, WS, BIG, None) == OK
    assert cand(ctypes.byref(d), ctypes.byref(c), 4, None, None, A, A, A, 8, A, 4, WS, BIG, None) == INVALID  # ld < n
    assert cand(ctypes.byref(d), ctypes.byref(c), 4, None, None, A, A, None, 8, A, 8, WS, BIG, None) == INVALID
    assert cand(ctypes.byref(d), ctypes.byref(c), 70000, A, None, A, A, A, 8, A, 8, WS, BIG, None) == UNSUPPORTED
    two = lsa.lib().lsa_two_stage_select
    k = d.top_k
    assert two(ctypes.byref(d), ctypes.byref(c), A, A, 4, None, None, A, A, k - 1, A, WS, BIG, None) == INVALID
    assert two(ctypes.byref(d), ctypes.byref(c), MISALIGNED, A, 4, None, None, A, A, k, A, WS, BIG, None) == INVALID
    fp8 = _dims(synth.DECODE_B4_FP8)
    cf = _cache(fp8)
    assert two(ctypes.byref(fp8), ctypes.byref(cf), A, A, 4, None, None, A, A, fp8.top_k, A, WS, BIG,
               None) == UNSUPPORTED                               # the original keys must be bf16
    assert lsa.lib().lsa_two_stage_workspace_size(ctypes.byref(d), 4, 4096, k - 1) == 0


def test_block_selection_checks():
    sel = lsa.lib().lsa_block_select
    assert sel(A, 4096, 0, A, 4096, 64, 8, A, WS, BIG, None) == OK
    assert sel(A, 4096, 4, A, 4096, 0, 8, A, WS, BIG, None) == INVALID     # block size
    assert sel(A, 4096, 4, A, 4096, 64, 0, A, WS, BIG, None) == INVALID    # blocks to keep
    assert sel(A, 4092, 4, A, 4096, 64, 8, A, WS, BIG, None) == INVALID    # ld below n_cols
    assert sel(A, 4096, 4, A, 4096, 64, 8, None, WS, BIG, None) == INVALID
    assert sel(A, 4096, 70000, A, 4096, 64, 8, A, WS, BIG, None) == UNSUPPORTED
    assert sel(A, 4096, 4, A, 4096, 64, 8, A, WS, 16, None) == WORKSPACE
    d = _dims()
    c = _cache(d)
    stage = lsa.lib().lsa_stage_blocks
    assert stage(ctypes.byref(d), ctypes.byref(c), 0, None, None, A, 8, 64, A, A, A, WS, BIG, None) == OK
    assert stage(ctypes.byref(d), ctypes.byref(c), 4, None, None, A, 8, 32, A, A, A, WS, BIG, None) == INVALID  # not one page
    assert stage(ctypes.byref(d), ctypes.byref(c), 4, None, None, A, 0, 64, A, A, A, WS, BIG, None) == INVALID
    assert stage(ctypes.byref(d), ctypes.byref(c), 4, None, None, A, 8, 64, MISALIGNED, A, A, WS, BIG,
                 None) == INVALID
    assert stage(ctypes.byref(d), ctypes.byref(c), 70000, A, None, A, 8, 64, A, A, A, WS, BIG, None) == UNSUPPORTED


def test_prefill_layers_checks():
    d = _dims(synth.PREFILL)
    assert d.block_size == 0
    c = _cache(d, batch=1, max_len=8192)
    arr = (lsa.Cache * 1)(c)
    P = lambda v: (ctypes.c_void_p * 1)(v)
    ev = (ctypes.c_void_p * 4)(A, A, A, A)
    kvb = (ctypes.c_void_p * 2)(A, A)
    call = lambda dd=d, rows=256, hist=4096, row_block=128, kv_buf=kvb, chunk=P(A): lsa.lib().lsa_prefill_layers(
        ctypes.byref(dd), 1, arr, hist, chunk, rows, A, P(A), P(A), P(A), P(A), None, None, row_block, kv_buf, WS,
        BIG, None, None, ev)
    assert call(rows=0) == OK
    assert call(dd=_dims(synth.DECODE_B32)) == INVALID            # paged: the history must be contiguous
    assert call(hist=9000) == INVALID                             # history longer than the cache
    assert call(row_block=0) == INVALID
    assert call(chunk=None) == INVALID                            # the chunk's own keys and rows are needed
    assert call(kv_buf=(ctypes.c_void_p * 2)(A, MISALIGNED)) == INVALID
    assert call(rows=70000) == UNSUPPORTED
