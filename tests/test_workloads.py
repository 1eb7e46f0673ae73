"""Host logic of the workload table and the bench's use of it (no GPU)."""
import pytest

import bench
from sparse_attention_decode_scan_b200 import synth


def test_names_and_prefixes_resolve():
    for name, spec in synth.WORKLOADS.items():
        assert spec.name == name and synth.workload(name) is spec
    assert synth.workload("decode_B32").name == synth.DECODE_B32
    assert synth.workload("prefill").name == synth.PREFILL
    with pytest.raises(KeyError):
        synth.workload("decode")          # several decode workloads
    with pytest.raises(KeyError):
        synth.workload("no_such_workload")


def test_seeds_are_distinct_per_workload_and_rank():
    seeds = {bench.rank_seed(s, r) for s in synth.WORKLOADS.values() for r in range(8)}
    assert len(seeds) == len(synth.WORKLOADS) * 8


def test_l2_flush_rule():
    # the key stream of a step exceeds twice the L2 only for the large decode batches
    want = {synth.TINY: False, synth.DECODE_B1: False, synth.DECODE_B32: True, synth.DECODE_B4_FP8: True,
            synth.PREFILL: False}
    assert {n: s.streams_past_l2 for n, s in synth.WORKLOADS.items()} == want


def test_layer_queries_match_the_layer_cases():
    import numpy as np
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=2, len_lo=100, len_hi=300, n_idx_heads=4,
                        idx_dim=16, n_heads=4, qk_dim=32, v_dim=16, top_k=16)
    for layer in (0, 3):
        c = synth.make_case(spec, 51, layer=layer)
        q_idx, w, q = synth.queries(spec, 51, c.rows, layer=layer)
        assert np.array_equal(q_idx, c.q_idx) and np.array_equal(w, c.w) and np.array_equal(q, c.q)
