"""Pins of the oracle's block selection (SparDA abstract, page 4 of the sources:
the selector picks the KV blocks a layer needs).  A block's score is the largest
indexer score of its visible tokens; the best n blocks are kept, ties to the
lower block; the layer attends every visible token of the kept blocks."""
import itertools

import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth


def test_hand_example():
    sc = np.array([1.0, 5.0, 2.0, 2.0, 9.0, 0.0, 3.0, 3.0])
    assert O.block_scores(sc, 8, 2).tolist() == [5.0, 2.0, 9.0, 3.0]
    assert O.block_select(sc, 8, 2, 2).tolist() == [0, 2]
    assert O.block_select(sc, 8, 2, 3).tolist() == [0, 2, 3]
    assert O.block_positions(np.array([0, 2]), 2, 8).tolist() == [0, 1, 4, 5]


def test_ties_go_to_the_lower_block_and_padding():
    sc = np.array([1.0, 1.0, 1.0, 1.0, 1.0, 1.0])
    assert O.block_select(sc, 6, 2, 2).tolist() == [0, 1]
    assert O.block_select(sc, 6, 2, 5).tolist() == [0, 1, 2, -1, -1]


def test_valid_length_cuts_the_last_block():
    sc = np.array([1.0, 2.0, 3.0, 4.0, 9.0, 9.0])
    # position 4 and 5 are not visible: block 2 has no visible token
    assert O.block_scores(sc, 4, 2).tolist() == [2.0, 4.0]
    assert O.block_select(sc, 4, 2, 1).tolist() == [1]
    # a partial last block keeps only its visible positions
    assert O.block_scores(sc, 5, 2).tolist() == [2.0, 4.0, 9.0]
    assert O.block_positions(np.array([2]), 2, 5).tolist() == [4]


def test_masked_entries_never_make_a_block():
    sc = np.array([-np.inf, -np.inf, 0.5, np.nan, -np.inf, np.nan])
    assert O.block_scores(sc, 6, 2).tolist() == [-np.inf, 0.5, -np.inf]
    assert O.block_select(sc, 6, 2, 3).tolist() == [1, -1, -1]


def test_block_size_one_is_the_token_top_k():
    g = np.random.default_rng(3)
    for n, k in [(50, 7), (9, 9), (30, 40)]:
        sc = g.integers(-3, 4, n).astype(np.float64)
        assert np.array_equal(O.block_select(sc, n, 1, k), O.topk(sc, n, k))


def test_kept_blocks_dominate_and_hold_the_best_token():
    """Brute force on small rows: the kept set is the lexicographically best
    set (block score descending, block index ascending) of its size."""
    g = np.random.default_rng(11)
    for _ in range(200):
        n = int(g.integers(1, 13))
        bs = int(g.integers(1, 4))
        L = int(g.integers(0, n + 1))
        sc = g.integers(-2, 3, n).astype(np.float64)
        nb = (L + bs - 1) // bs
        kk = int(g.integers(1, 5))
        got = [b for b in O.block_select(sc, L, bs, kk).tolist() if b >= 0]
        bscore = [max(sc[b * bs:min((b + 1) * bs, L)]) for b in range(nb)]
        best = min(itertools.combinations(range(nb), min(kk, nb)),
                   key=lambda c: sorted((-bscore[b], b) for b in c))
        assert got == sorted(best)
        if L > 0:
            top_token = int(O.topk(sc, L, 1)[0])
            assert top_token // bs in got


def test_row_block_step_covers_the_kept_blocks():
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=2, len_lo=300, len_hi=700, n_idx_heads=4,
                        idx_dim=16, n_heads=4, qk_dim=32, v_dim=16, top_k=8)
    case = synth.make_case(spec, 5)
    for r in range(case.rows):
        L = O.row_visible(case, r)
        blocks, pos, o, lse = O.row_block_step(case, r, 4)
        kept = [b for b in blocks if b >= 0]
        assert len(kept) == min(4, (L + spec.block_size - 1) // spec.block_size)
        assert all(p // spec.block_size in kept and p < L for p in pos)
        assert len(pos) == sum(min(spec.block_size, L - b * spec.block_size) for b in kept)
        o2, l2 = O.row_attention(case, r, pos)
        assert np.allclose(o, o2) and np.allclose(lse, l2)
