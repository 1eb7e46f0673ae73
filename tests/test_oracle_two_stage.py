"""Pins of the oracle's two-stage indexer search (LeanSparse episode page,
summary paragraph: search compact keys, fetch a short list of originals and
rank them exactly)."""
import numpy as np

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth


def _tiny_case(keys, q, w):
    """One sequence, fp32 keys and queries of the given values."""
    L, d = keys.shape
    spec = synth.Spec("hand", batch=1, len_lo=L, len_hi=L, n_idx_heads=q.shape[0], idx_dim=d, n_heads=1,
                      qk_dim=8, v_dim=8, top_k=1, act_dtype="f32", idx_key_dtype="f32", with_kv=False)
    return synth.Case(spec, 0, np.array([L], np.int32), None, keys.astype(np.float32)[None], None, None,
                      np.array([0], np.int32), None, q.astype(np.float32)[None], w.astype(np.float32)[None], None)


def test_hand_example_the_short_list_decides():
    # exact scores (1, 2, 3); compact scores (3, 2, 1): the two best by the
    # compact keys are tokens 0 and 1, and token 1 ranks first among them
    case = _tiny_case(np.array([[1.0], [2.0], [3.0]]), np.array([[1.0]]), np.array([1.0]))
    bits = np.array([[[0x44], [0x40], [0x38]]], np.uint8)   # e4m3 3.0, 2.0, 1.0
    scales = np.ones((1, 3), np.float32)
    assert O.e4m3_to_f64(bits).ravel().tolist() == [3.0, 2.0, 1.0]
    assert O.two_stage_select(case, bits, scales, 0, 1, 2).tolist() == [1]
    assert O.two_stage_select(case, bits, scales, 0, 2, 2).tolist() == [0, 1]
    # a list as long as the sequence gives the exact top-k
    assert O.two_stage_select(case, bits, scales, 0, 1, 3).tolist() == [2]
    assert O.topk(O.row_scores(case, 0), 3, 1).tolist() == [2]


def _spec():
    return synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=3, len_lo=200, len_hi=600, n_idx_heads=4,
                        idx_dim=16, top_k=32, with_kv=False)


def test_full_length_list_is_the_exact_top_k():
    case = synth.make_case(_spec(), 41)
    bits, scales = synth.compact_keys(case.idx_keys)
    for r in range(case.rows):
        L = O.row_visible(case, r)
        exact = O.topk(O.row_scores(case, r), L, 32)
        assert np.array_equal(O.two_stage_select(case, bits, scales, r, 32, L), exact)


def test_lossless_compact_keys_give_the_exact_top_k_for_any_list_length():
    case = synth.make_case(_spec(), 42)
    # small-integer keys: exact in bf16 and in e4m3 with scale 1 (many ties)
    rng = synth.rng(42, "int_keys")
    ints = rng.integers(-4, 5, size=case.idx_keys.shape).astype(np.float32)
    case.idx_keys[...] = synth.to_bf16_bits(ints)
    bits = synth.to_e4m3_bits(ints)
    scales = np.ones(ints.shape[:-1], np.float32)
    for r in range(case.rows):
        L = O.row_visible(case, r)
        exact = O.topk(O.row_scores(case, r), L, 32)
        for n_cand in (32, 33, 64, L):
            assert np.array_equal(O.two_stage_select(case, bits, scales, r, 32, n_cand), exact)


def test_selection_comes_from_the_short_list():
    case = synth.make_case(_spec(), 43)
    bits, scales = synth.compact_keys(case.idx_keys)
    for r in range(case.rows):
        L = O.row_visible(case, r)
        cand = set(O.topk(O.compact_row_scores(case, bits, scales, r), L, 64).tolist()) - {-1}
        sel = O.two_stage_select(case, bits, scales, r, 32, 64)
        got = [int(x) for x in sel if x >= 0]
        assert len(got) == min(32, L) and set(got) <= cand
        # the k best candidates by their exact scores
        exact = O.row_scores(case, r)
        worst_in = min(exact[got])
        assert all(exact[c] <= worst_in for c in cand - set(got))


def test_compact_keys_round_trip_within_e4m3_precision():
    case = synth.make_case(_spec(), 44)
    bits, scales = synth.compact_keys(case.idx_keys)
    full = O.bf16_to_f64(case.idx_keys)
    back = O.e4m3_to_f64(bits) * scales[..., None]
    amax = np.abs(full).max(axis=-1, keepdims=True)
    # e4m3 keeps 3 mantissa bits: half an ulp is 2^-4 relative; subnormals of
    # the scaled range add at most 2^-10 of the token's largest magnitude
    assert np.all(np.abs(back - full) <= np.abs(full) * 2.0 ** -4 + amax * 2.0 ** -9)
