"""Pins of the oracle's multi-layer routing ("Multi-layer Indexer" abstract,
zhuanzhiai.com, sentences 4-5 and 8-9): which selection each layer attends
under IndexCache (ROUTE_OWN) and under MLI (ROUTE_PREV), and what the layers
compute with it."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth


# Hand tables from the definitions: indexer layers 0, r, 2r, ...; IndexCache
# attends the latest indexer layer at or before the layer, MLI the latest one
# strictly before it (layer 0 its own).
@pytest.mark.parametrize("n,r,own,prev", [
    (1, 1, [0], [0]),
    (4, 1, [0, 1, 2, 3], [0, 0, 1, 2]),
    (6, 2, [0, 0, 2, 2, 4, 4], [0, 0, 0, 2, 2, 4]),
    (5, 4, [0, 0, 0, 0, 4], [0, 0, 0, 0, 0]),
    (7, 3, [0, 0, 0, 3, 3, 3, 6], [0, 0, 0, 0, 3, 3, 3]),
])
def test_selection_source_tables(n, r, own, prev):
    assert O.indexer_layers(n, r) == list(range(0, n, r))
    assert O.selection_source(n, r, O.ROUTE_OWN) == own
    assert O.selection_source(n, r, O.ROUTE_PREV) == prev


def _spec():
    return synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=3, len_lo=60, len_hi=300, n_idx_heads=4,
                        idx_dim=16, n_heads=4, qk_dim=32, v_dim=16, top_k=48, softmax_scale=0.25)


def test_one_layer_is_the_single_step():
    case = synth.make_case(_spec(), 31)
    for route in (O.ROUTE_OWN, O.ROUTE_PREV):
        src, res = O.decode_layers([case], 1, route)
        assert src == [0]
        idx, o, lse = res[0]
        for r in range(case.rows):
            _, sel, o_r, l_r = O.row_step(case, r)
            assert np.array_equal(idx[r], sel)
            np.testing.assert_array_equal(o[r], o_r)
            np.testing.assert_array_equal(lse[r], l_r)


def test_identical_layers_make_the_routes_agree():
    case = synth.make_case(_spec(), 32)
    _, own = O.decode_layers([case] * 3, 1, O.ROUTE_OWN)
    _, prev = O.decode_layers([case] * 3, 1, O.ROUTE_PREV)
    for a, b in zip(own, prev):
        for x, y in zip(a, b):
            np.testing.assert_array_equal(x, y)


def test_mli_layer_attends_the_previous_layers_own_selection_with_its_own_query_and_cache():
    layers = synth.make_layers(_spec(), 33, 3)
    _, own = O.decode_layers(layers, 1, O.ROUTE_OWN)
    _, prev = O.decode_layers(layers, 1, O.ROUTE_PREV)
    # the layers differ, so their own selections differ
    assert not np.array_equal(own[1][0], own[0][0])
    for l in (1, 2):
        assert np.array_equal(prev[l][0], own[l - 1][0])
        c = layers[l]
        for r in range(c.rows):
            o_r, l_r = O.row_attention(c, r, own[l - 1][0][r])
            np.testing.assert_array_equal(prev[l][1][r], o_r)
            np.testing.assert_array_equal(prev[l][2][r], l_r)
            # not the source layer's query or cache
            o_src, _ = O.row_attention(layers[l - 1], r, own[l - 1][0][r])
            assert not np.allclose(prev[l][1][r], o_src)


def test_layers_share_lengths_and_pages_but_not_contents():
    layers = synth.make_layers(_spec(), 34, 2)
    a, b = layers
    assert np.array_equal(a.seq_lens, b.seq_lens) and np.array_equal(a.block_table, b.block_table)
    assert not np.array_equal(a.idx_keys, b.idx_keys) and not np.array_equal(a.kv, b.kv)
    assert not np.array_equal(a.q_idx, b.q_idx) and not np.array_equal(a.q, b.q)
    # layer 0 is the plain single-layer case
    c = synth.make_case(_spec(), 34)
    assert np.array_equal(a.idx_keys, c.idx_keys) and np.array_equal(a.q, c.q)
