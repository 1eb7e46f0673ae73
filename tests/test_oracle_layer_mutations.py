"""Plant plausible mistakes in the oracle's multi-layer routing and two-stage
search (on the CPU) and check that the pins catch each one."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from tests import test_oracle_layers as PL
from tests import test_oracle_two_stage as PT

_orig_source = O.selection_source
_orig_row_attention = O.row_attention


def _source_prev_inclusive(n, r, route):
    # MLI taken as "at or before", the IndexCache rule
    return _orig_source(n, r, O.ROUTE_OWN)


def _source_indexers_shifted(n, r, route):
    # indexer layers r-1, 2r-1, ... instead of 0, r, 2r, ...
    keep = [l for l in range(n) if (l + 1) % r == 0] or [0]
    src = []
    for l in range(n):
        before = [i for i in keep if (i <= l if route == O.ROUTE_OWN else i < l)]
        src.append(before[-1] if before else 0)
    return src


def _layers_source_query(layers, retention, route):
    # the layer attends with the source layer's query and cache
    src = _orig_source(len(layers), retention, route)
    res = []
    for l, c in enumerate(layers):
        s = layers[src[l]]
        idx = np.stack([O.topk(O.row_scores(s, r), O.row_visible(s, r), s.spec.top_k) for r in range(s.rows)])
        att = [_orig_row_attention(s, r, idx[r]) for r in range(c.rows)]
        res.append((idx, np.stack([a[0] for a in att]), np.stack([a[1] for a in att])))
    return src, res


def _two_stage_compact_ranking(case, bits, scales, r, k, n_cand):
    L = O.row_visible(case, r)
    return O.topk(O.compact_row_scores(case, bits, scales, r), L, k)


def _two_stage_exact_candidates(case, bits, scales, r, k, n_cand):
    L = O.row_visible(case, r)
    return O.topk(O.row_scores(case, r), L, k)


def _two_stage_list_of_k(case, bits, scales, r, k, n_cand):
    return _orig_two_stage(case, bits, scales, r, k, k)


_orig_two_stage = O.two_stage_select

MUTANTS = {
    "source_prev_inclusive": ("selection_source", _source_prev_inclusive),
    "source_indexers_shifted": ("selection_source", _source_indexers_shifted),
    "layers_source_query": ("decode_layers", _layers_source_query),
    "two_stage_compact_ranking": ("two_stage_select", _two_stage_compact_ranking),
    "two_stage_exact_candidates": ("two_stage_select", _two_stage_exact_candidates),
    "two_stage_list_of_k": ("two_stage_select", _two_stage_list_of_k),
}


def _run_pins():
    checks = [lambda a=a: PL.test_selection_source_tables(*a) for a in [
        (1, 1, [0], [0]), (4, 1, [0, 1, 2, 3], [0, 0, 1, 2]), (6, 2, [0, 0, 2, 2, 4, 4], [0, 0, 0, 2, 2, 4]),
        (5, 4, [0, 0, 0, 0, 4], [0, 0, 0, 0, 0]), (7, 3, [0, 0, 0, 3, 3, 3, 6], [0, 0, 0, 0, 3, 3, 3])]]
    checks += [PL.test_one_layer_is_the_single_step, PL.test_identical_layers_make_the_routes_agree,
               PL.test_mli_layer_attends_the_previous_layers_own_selection_with_its_own_query_and_cache,
               PT.test_hand_example_the_short_list_decides, PT.test_full_length_list_is_the_exact_top_k,
               PT.test_lossless_compact_keys_give_the_exact_top_k_for_any_list_length,
               PT.test_selection_comes_from_the_short_list]
    failures = 0
    for chk in checks:
        try:
            chk()
        except Exception:
            failures += 1
    return failures


def test_unmutated_oracle_passes_every_pin():
    assert _run_pins() == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(O, attr, fn)
    assert _run_pins() > 0, f"mutant {name} survived every pin"
