"""Indexer scores on the GPU vs the oracle (both GPU paths)."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests import cases
from tests.helpers import SCORE_TOL, check_scores

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _run_scores(case, monkeypatch=None):
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(case)
    rows = dc.rows
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.full((rows, ld), 7.0, dtype=torch.float32, device="cuda")  # sentinel
    ws = lsa.workspace(lsa.workspace_size(dc.dims, rows, dc.max_len, lsa.LSA_OP_SCORES))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq,
                       row_pos=dc.row_pos)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    return scores.cpu().numpy()


def _check_rows(case, scores, rows):
    tol = SCORE_TOL[case.spec.idx_key_dtype]
    for r in rows:
        L = int(case.seq_lens[case.row_seq[r]])
        ref = O.row_scores(case, r)
        check_scores(scores[r, :L], ref, tol, what=f"{case.spec.name} row {r}")
        assert np.isneginf(scores[r, L:]).all(), f"row {r}: tail past the sequence is not -inf"


@pytest.mark.parametrize("path", ["default", "simt"])
@pytest.mark.parametrize("name", list(cases.SMALL))
def test_scores_small(name, path, request):
    if path == "simt":
        request.getfixturevalue("test_hooks")(force_simt=True)
    case = cases.small(name)
    scores = _run_scores(case)
    _check_rows(case, scores, range(case.rows))


@pytest.mark.slow
@pytest.mark.parametrize("name", [synth.DECODE_B1, synth.DECODE_B32, synth.DECODE_B4_FP8])
def test_scores_full_decode(name):
    case = cases.full(name, with_kv=False)
    scores = _run_scores(case)
    rows = sorted({0, case.rows - 1, case.rows // 2})
    _check_rows(case, scores, rows)
    # every row: tails are -inf and visible entries finite
    for r in range(case.rows):
        L = int(case.seq_lens[r])
        assert np.isfinite(scores[r, :L]).all() and np.isneginf(scores[r, L:]).all()


@pytest.mark.slow
def test_scores_full_prefill():
    case = cases.full(synth.PREFILL, with_kv=False)
    scores = _run_scores(case)
    g = np.random.default_rng(77)
    rows = sorted({0, 1, case.rows - 2, case.rows - 1, *g.integers(0, case.rows, 4).tolist()})
    _check_rows(case, scores, rows)
