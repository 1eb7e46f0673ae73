"""Plant plausible mistakes in the oracle (on the CPU) and check the pins catch each.

Every mutant below must make at least one pin of test_oracle_pins fail; a
mutant that survives means the pins leave that part of the oracle unchecked.
"""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from tests import test_oracle_pins as P

_orig_scores = O.indexer_scores
_orig_topk = O.topk
_orig_attn = O.attention


def _scores_no_relu(q, w, keys, scales=None, pos=None):
    dots = np.asarray(keys, float) @ np.asarray(q, float).T
    if scales is not None:
        dots = dots * np.asarray(scales, float)[:, None]
    s = dots @ np.asarray(w, float)
    if pos is not None:
        s[int(pos) + 1:] = -np.inf
    return s


def _scores_relu_after_weight(q, w, keys, scales=None, pos=None):
    dots = np.asarray(keys, float) @ np.asarray(q, float).T
    if scales is not None:
        dots = dots * np.asarray(scales, float)[:, None]
    s = np.maximum(dots * np.asarray(w, float)[None, :], 0).sum(1)
    if pos is not None:
        s[int(pos) + 1:] = -np.inf
    return s


def _scores_transposed_q(q, w, keys, scales=None, pos=None):
    q = np.asarray(q, float)
    if q.shape[0] == q.shape[1]:
        q = q.T
    return _orig_scores(q, w, keys, scales, pos)


def _scores_scale_dropped(q, w, keys, scales=None, pos=None):
    return _orig_scores(q, w, keys, None, pos)


def _scores_causal_off_by_one(q, w, keys, scales=None, pos=None):
    return _orig_scores(q, w, keys, scales, None if pos is None else pos - 1)


def _topk_high_index_ties(scores, valid_len, k):
    s = np.asarray(scores)[:int(valid_len)]
    pos = np.arange(s.shape[0])
    ok = ~(np.isnan(s) | (s == -np.inf))
    order = np.lexsort((-pos[ok], -s[ok]))
    take = np.sort(pos[ok][order[:k]])
    out = np.full(k, -1, np.int32)
    out[:take.shape[0]] = take
    return out


def _topk_keeps_neg_inf(scores, valid_len, k):
    s = np.asarray(scores)[:int(valid_len)]
    pos = np.arange(s.shape[0])
    order = np.lexsort((pos, -s))
    take = np.sort(pos[order[:k]])
    out = np.full(k, -1, np.int32)
    out[:take.shape[0]] = take
    return out


def _topk_descending_output(scores, valid_len, k):
    out = _orig_topk(scores, valid_len, k)
    n = int((out >= 0).sum())
    out[:n] = out[:n][::-1]
    return out


def _attn_no_scale(q, kv_rows, v_dim, scale):
    return _orig_attn(q, kv_rows, v_dim, 1.0)


def _attn_tail_values(q, kv_rows, v_dim, scale):
    kv = np.asarray(kv_rows, float)
    o, lse = _orig_attn(q, kv, kv.shape[1], scale)
    return o[:, -v_dim:], lse


def _attn_lse_without_max(q, kv_rows, v_dim, scale):
    o, lse = _orig_attn(q, kv_rows, v_dim, scale)
    z = scale * np.asarray(q, float) @ np.asarray(kv_rows, float).T
    return o, np.log(np.exp(z - z.max(1, keepdims=True)).sum(1))


MUTANTS = {
    "scores_no_relu": ("indexer_scores", _scores_no_relu),
    "scores_relu_after_weight": ("indexer_scores", _scores_relu_after_weight),
    "scores_transposed_q": ("indexer_scores", _scores_transposed_q),
    "scores_scale_dropped": ("indexer_scores", _scores_scale_dropped),
    "scores_causal_off_by_one": ("indexer_scores", _scores_causal_off_by_one),
    "topk_high_index_ties": ("topk", _topk_high_index_ties),
    "topk_keeps_neg_inf": ("topk", _topk_keeps_neg_inf),
    "topk_descending_output": ("topk", _topk_descending_output),
    "attn_no_scale": ("attention", _attn_no_scale),
    "attn_tail_values": ("attention", _attn_tail_values),
    "attn_lse_without_max": ("attention", _attn_lse_without_max),
}


def _run_pins():
    """Run the deterministic pins; return the number that failed."""
    failures = 0
    checks = []
    for c in P._load("indexer_hand.json")["cases"]:
        checks.append(lambda c=c: P.test_indexer_hand_examples(c))
    for c in P._load("attention_hand.json")["cases"]:
        checks.append(lambda c=c: P.test_attention_hand_examples(c))
    checks += [P.test_indexer_single_head_unit_weight_is_relu_dot, P.test_indexer_positive_scale_invariance,
               P.test_topk_distinct_matches_argpartition, P.test_topk_negative_zero_equals_positive_zero,
               P.test_attention_matches_torch_sdpa, P.test_attention_invariants,
               P.test_prefill_rows_are_causal, P.test_selection_size_and_distinctness]
    checks += [lambda s=s: P.test_topk_brute_force_tiny(s) for s in range(40)]
    for chk in checks:
        try:
            chk()
        except AssertionError:
            failures += 1
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
