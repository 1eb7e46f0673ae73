"""Host-side argument checks of lsa_decode_layers: refused before any CUDA
call, so they run without a GPU (fake, aligned device addresses)."""
import ctypes

from sparse_attention_decode_scan_b200 import lsa, synth
from sparse_attention_decode_scan_b200.device import make_dims


def _cache(seq_lens=0x40000, batch=3, max_len=2560):
    c = lsa.Cache()
    c.idx_keys, c.idx_key_scales, c.kv, c.block_table = 0x10000, None, 0x20000, 0x30000
    c.max_blocks_per_seq, c.n_blocks, c.max_len, c.seq_lens, c.batch = 40, 100, max_len, seq_lens, batch
    return c


def _call(caches, retention=1, route=lsa.LSA_ROUTE_PREV, q_idx=0x50000, n=None):
    d = make_dims(synth.scaled(synth.WORKLOADS[synth.DECODE_B32], top_k=256))
    n = len(caches) if n is None else n
    arr = (lsa.Cache * max(len(caches), 1))(*caches)
    P = lambda v: (ctypes.c_void_p * max(len(caches), 1))(*([v] * max(len(caches), 1)))
    return lsa.lib().lsa_decode_layers(ctypes.byref(d), n, arr, P(q_idx), P(0x60000), P(0x70000), P(0x80000),
                                       None, retention, route, None, ctypes.c_void_p(0x1000000), 1 << 34, None)


def test_bad_counts_and_routes():
    assert _call([_cache()], n=0) == lsa.LSA_ERR_INVALID_ARG
    assert _call([_cache()], retention=0) == lsa.LSA_ERR_INVALID_ARG
    assert _call([_cache()], route=7) == lsa.LSA_ERR_INVALID_ARG


def test_layers_must_share_the_batch_layout():
    assert _call([_cache(), _cache(seq_lens=0x41000)]) == lsa.LSA_ERR_INVALID_ARG
    assert _call([_cache(), _cache(batch=2)]) == lsa.LSA_ERR_INVALID_ARG
    assert _call([_cache(), _cache(max_len=2624)]) == lsa.LSA_ERR_INVALID_ARG


def test_indexer_layers_need_their_queries():
    assert _call([_cache(), _cache()], q_idx=0) == lsa.LSA_ERR_INVALID_ARG
    assert _call([_cache(), _cache()], q_idx=0x50008) == lsa.LSA_ERR_INVALID_ARG  # misaligned
