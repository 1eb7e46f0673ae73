"""Pins of the CPU oracle to things other than itself (no GPU needed).

Hand-worked examples (tests/golden), closed forms, library routines
(torch's bf16/e4m3 decoders, scaled_dot_product_attention, numpy
argpartition), brute force on tiny inputs and invariants.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _num(v):
    return -np.inf if v == "-inf" else (np.nan if v == "nan" else float(v))


# --------------------------------------------------------------------------- decoders

def test_bf16_decode_matches_torch_all_codes():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    ours = O.bf16_to_f64(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()
    assert np.array_equal(np.signbit(ours[~np.isnan(ours)]), np.signbit(ref[~np.isnan(ref)]))


def test_e4m3_decode_matches_torch_all_codes():
    bits = np.arange(256, dtype=np.uint8)
    ours = O.e4m3_to_f64(bits)
    ref = torch.from_numpy(bits).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


def test_e4m3_decode_spec_points():
    g = _load("e4m3_points.json")
    for code, val in g["points"]:
        got = O.e4m3_to_f64(np.array([int(code, 16)], np.uint8))[0]
        want = _num(val)
        if np.isnan(want):
            assert np.isnan(got), code
        else:
            assert got == want and np.signbit(got) == np.signbit(want), code


def test_synth_encoders_round_trip_nearest():
    # the generator's encoders must round to the nearest representable value
    x = synth.normal((4096,), 7, "rt") * np.float32(3.0)
    b = O.bf16_to_f64(synth.to_bf16_bits(x))
    e = O.e4m3_to_f64(synth.to_e4m3_bits(x))
    assert np.all(np.abs(b - x) <= np.abs(x) * 2.0 ** -8 + 1e-30)
    assert np.all(np.abs(e - x) <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10) + 1e-12)


# --------------------------------------------------------------------------- indexer

@pytest.mark.parametrize("case", _load("indexer_hand.json")["cases"], ids=lambda c: c["name"])
def test_indexer_hand_examples(case):
    scales = case.get("scales")
    got = O.indexer_scores(np.array(case["q"], float), np.array(case["w"], float),
                           np.array(case["keys"], float),
                           None if scales is None else np.array(scales, float), case.get("pos"))
    want = np.array([_num(v) for v in case["scores"]])
    assert np.array_equal(got, want)
    sel = O.topk(got, got.shape[0], case["k"])
    assert sel.tolist() == case["topk"]


def test_indexer_single_head_unit_weight_is_relu_dot():
    g = np.random.default_rng(3)
    q = g.standard_normal((1, 16))
    keys = g.standard_normal((50, 16))
    got = O.indexer_scores(q, np.ones(1), keys)
    want = np.array([max(0.0, float(np.dot(q[0], k))) for k in keys])
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_indexer_positive_scale_invariance():
    g = np.random.default_rng(4)
    q, w, keys = g.standard_normal((8, 32)), g.standard_normal(8), g.standard_normal((40, 32))
    sc = g.uniform(0.5, 2.0, 40)
    a = O.indexer_scores(q, w, keys, sc)
    b = O.indexer_scores(q, w, keys * sc[:, None])
    c = O.indexer_scores(q, w, keys) * sc
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12) and np.allclose(a, c, rtol=1e-12, atol=1e-12)


def test_indexer_head_additivity():
    # splitting the heads into two groups and summing gives the same scores
    g = np.random.default_rng(5)
    q, w, keys = g.standard_normal((6, 8)), g.standard_normal(6), g.standard_normal((30, 8))
    full = O.indexer_scores(q, w, keys)
    parts = O.indexer_scores(q[:2], w[:2], keys) + O.indexer_scores(q[2:], w[2:], keys)
    assert np.allclose(full, parts, rtol=1e-12, atol=1e-12)


def test_paged_addressing_hand_example():
    # block size 2, sequence 0 owns physical blocks 2 then 0
    bt = np.array([[2, 0]], np.int32)
    rows = O.physical_rows(0, np.arange(4), bt, 2, 0)
    assert rows.tolist() == [4, 5, 0, 1]
    assert O.physical_rows(1, np.arange(3), None, 0, 10).tolist() == [10, 11, 12]


def test_paged_equals_contiguous_on_synthetic_case():
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=2, len_lo=150, len_hi=300, n_idx_heads=4,
                        idx_dim=16, n_heads=4, qk_dim=24, v_dim=16, top_k=32, block_size=16)
    case = synth.make_case(spec, 11)
    # rebuild the same logical cache contiguously
    stride = spec.len_hi
    keys_c = np.zeros((spec.batch, stride, spec.idx_dim), case.idx_keys.dtype)
    kv_c = np.zeros((spec.batch, stride, spec.qk_dim), case.kv.dtype)
    for b in range(spec.batch):
        L = int(case.seq_lens[b])
        keys_c[b, :L] = O.cache_rows(case.idx_keys, b, np.arange(L), case.block_table, 16, 0)
        kv_c[b, :L] = O.cache_rows(case.kv, b, np.arange(L), case.block_table, 16, 0)
    import dataclasses
    spec_c = dataclasses.replace(spec, block_size=0)
    case_c = dataclasses.replace(case, spec=spec_c, block_table=None, idx_keys=keys_c, kv=kv_c)
    for r in range(spec.batch):
        s1, i1, o1, l1 = O.row_step(case, r)
        s2, i2, o2, l2 = O.row_step(case_c, r)
        assert np.array_equal(s1, s2) and np.array_equal(i1, i2)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# --------------------------------------------------------------------------- top-k

def test_topk_distinct_matches_argpartition():
    g = np.random.default_rng(6)
    for n, k in [(1000, 37), (64, 64), (10, 20), (5000, 2048)]:
        s = g.permutation(n).astype(np.float32) * np.float32(0.5) - np.float32(7)
        want = np.sort(np.argpartition(-s, min(k, n) - 1)[:min(k, n)])
        got = O.topk(s, n, k)
        assert got[:min(k, n)].tolist() == want.tolist()
        assert (got[min(k, n):] == -1).all()


def _dominates(s, i, j):
    # i is preferred to j: higher score, or equal score and lower position
    return s[i] > s[j] or (s[i] == s[j] and i < j)


@pytest.mark.parametrize("seed", range(40))
def test_topk_brute_force_tiny(seed):
    g = np.random.default_rng(100 + seed)
    n = int(g.integers(1, 9))
    k = int(g.integers(1, 10))
    vals = np.array([0.0, -0.0, 1.0, -1.0, 2.5, -np.inf], np.float32)
    s = vals[g.integers(0, len(vals), n)]
    valid = int(g.integers(0, n + 1))
    got = O.topk(s, valid, k)
    selectable = [i for i in range(valid) if s[i] != -np.inf]
    m = min(k, len(selectable))
    # brute force: the unique m-subset whose members all dominate all non-members
    best = None
    for sub in itertools.combinations(selectable, m):
        rest = [j for j in selectable if j not in sub]
        if all(_dominates(s, i, j) for i in sub for j in rest):
            assert best is None
            best = sub
    assert best is not None
    assert got[:m].tolist() == sorted(best)
    assert (got[m:] == -1).all()


def test_topk_negative_zero_equals_positive_zero():
    s = np.array([-0.0, 0.0, -0.0, 0.0], np.float32)
    assert O.topk(s, 4, 2).tolist() == [0, 1]


def test_topk_compares_in_given_precision():
    # two fp32 values that differ only beyond fp32 precision are a tie
    a = np.float32(1.0)
    s = np.array([a, np.float32(1.0 + 1e-9), a], np.float32)
    assert O.topk(s, 3, 1).tolist() == [0]


# --------------------------------------------------------------------------- attention

@pytest.mark.parametrize("case", _load("attention_hand.json")["cases"], ids=lambda c: c["name"])
def test_attention_hand_examples(case):
    kv = np.array(case["kv"], float)
    idx = np.array(case["idx"])
    sel = idx[idx >= 0]
    o, lse = O.attention(np.array(case["q"], float), kv[sel], case["v_dim"], case["scale"])
    assert np.allclose(o, np.array(case["o"]), rtol=0, atol=1e-15)
    assert np.allclose(lse, np.array(case["lse"]), rtol=0, atol=1e-15)


def test_attention_matches_torch_sdpa():
    g = torch.Generator().manual_seed(9)
    H, n, D, Dv = 5, 33, 24, 16
    q = torch.randn(H, D, generator=g, dtype=torch.float64)
    kv = torch.randn(n, D, generator=g, dtype=torch.float64)
    scale = 0.3
    o, lse = O.attention(q.numpy(), kv.numpy(), Dv, scale)
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None, :, None, :], kv[None, None].expand(1, H, n, D), kv[None, None, :, :Dv].expand(1, H, n, Dv),
        scale=scale)[0, :, 0, :]
    ref_lse = torch.logsumexp(scale * (q @ kv.T), dim=1)
    assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-13)
    assert np.allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-13)


def test_sparse_with_k_at_least_L_equals_dense():
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B1], len_lo=200, len_hi=200, n_idx_heads=4, idx_dim=16,
                        n_heads=6, qk_dim=40, v_dim=32, top_k=256)
    case = synth.make_case(spec, 12)
    _, sel, o, lse = O.row_step(case, 0)
    assert (sel[:200] == np.arange(200)).all() and (sel[200:] == -1).all()
    q = torch.from_numpy(O.decode(case.q[0], "bf16"))
    kv = torch.from_numpy(O.decode(case.kv[0, :200], "bf16"))
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[None, :, None, :], kv[None, None].expand(1, 6, 200, 40), kv[None, None, :, :32].expand(1, 6, 200, 32),
        scale=spec.softmax_scale)[0, :, 0, :]
    assert np.allclose(o, ref.numpy(), rtol=0, atol=1e-12)


def test_attention_invariants():
    g = np.random.default_rng(8)
    q = g.standard_normal((4, 12))
    kv = g.standard_normal((20, 12))
    # weights sum to one: constant V rows give that constant back
    kv_c = kv.copy()
    kv_c[:, :8] = 3.25
    o, _ = O.attention(q, kv_c, 8, 0.5)
    assert np.allclose(o, 3.25, rtol=0, atol=1e-13)
    # every output coordinate lies within the range of its V column
    o, _ = O.attention(q, kv, 8, 0.5)
    assert (o >= kv[:, :8].min(0) - 1e-12).all() and (o <= kv[:, :8].max(0) + 1e-12).all()
    # lse is the log of the softmax normaliser
    z = 0.5 * q @ kv.T
    _, lse = O.attention(q, kv, 8, 0.5)
    assert np.allclose(np.exp(z - lse[:, None]).sum(1), 1.0, rtol=0, atol=1e-13)


# --------------------------------------------------------------------------- whole step invariants

def test_prefill_rows_are_causal():
    spec = synth.scaled(synth.WORKLOADS[synth.PREFILL], len_lo=300, len_hi=300, chunk=40, n_idx_heads=4, idx_dim=16,
                        n_heads=4, qk_dim=24, v_dim=16, top_k=64)
    case = synth.make_case(spec, 13)
    for r in [0, 17, 39]:
        sc, sel, o, lse = O.row_step(case, r)
        p = int(case.row_pos[r])
        assert np.isneginf(sc[p + 1:]).all() and np.isfinite(sc[:p + 1]).all()
        valid = sel[sel >= 0]
        assert len(valid) == min(64, p + 1) and len(set(valid.tolist())) == len(valid)
        assert (valid <= p).all()


def test_selection_size_and_distinctness():
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=3, len_lo=40, len_hi=300, n_idx_heads=4, idx_dim=16,
                        n_heads=4, qk_dim=24, v_dim=16, top_k=100, block_size=16)
    case = synth.make_case(spec, 14)
    for r in range(3):
        sc, sel, _, _ = O.row_step(case, r)
        L = int(case.seq_lens[r])
        valid = sel[sel >= 0]
        assert len(valid) == min(100, L) and len(np.unique(valid)) == len(valid)
        assert (np.diff(valid) > 0).all() and (valid < L).all()
        if L > 100:
            kth = np.sort(sc)[::-1][99]
            assert sc[valid].min() >= kth
