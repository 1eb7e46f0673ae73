"""The two-stage indexer search on the GPU (LeanSparse episode page, summary:
search compact keys, fetch a short list of the originals, rank them exactly)
against the oracle's two_stage_select, and its re-scoring stage against the
oracle's scores of the same positions."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests import cases
from tests.helpers import SCORE_TOL, SEL_TOL, check_scores

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _compact_device(case):
    bits, scales = synth.compact_keys(case.idx_keys)
    return bits, scales, torch.from_numpy(np.ascontiguousarray(bits)).cuda(), torch.from_numpy(scales).cuda()


def _cand_lists(case, n_cand, seed):
    vis = np.array([O.row_visible(case, r) for r in range(case.rows)], np.int64)
    return synth.index_lists(case.rows, n_cand, vis, seed)


@pytest.mark.parametrize("name,n_cand", [("bf16_L5000", 700), ("paged_B5", 1000), ("prefill_3000x256", 300),
                                         ("len1", 64)])
def test_candidate_scores_vs_oracle(name, n_cand):
    """Exact scores of given positions (several tiles and a ragged last tile,
    -1 padding where a row is shorter than the list)."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small(name)
    dc = DeviceCase(case)
    cand = _cand_lists(case, n_cand, 77)
    ld = (n_cand + 3) // 4 * 4 + 4
    out = torch.full((dc.rows, ld), 7.0, dtype=torch.float32, device="cuda")
    ws = lsa.workspace(256)
    lsa.candidate_scores(dc.dims, dc.cache, dc.q_idx, dc.w, torch.from_numpy(cand).cuda(), out, ld, ws,
                         row_seq=dc.row_seq, row_pos=dc.row_pos)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    got = out.cpu().numpy()
    rows = range(dc.rows) if dc.rows <= 8 else [0, 1, 77, dc.rows - 1]
    for r in rows:
        sc = O.row_scores(case, r)
        live = cand[r] >= 0
        ref = np.where(live, sc[np.where(live, cand[r], 0)], -np.inf)
        check_scores(got[r, :n_cand], ref, SCORE_TOL["bf16"], what=f"{name} row {r}")
        assert np.isneginf(got[r, n_cand:]).all()


def _int_case(seed):
    """Integer-valued keys, queries and weights: every score is an exact
    integer in fp32 and e4m3 holds the keys exactly (scale 1), so the compact
    and exact scores coincide on both sides and the selection is bit-exact,
    ties (many) included."""
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=3, len_lo=1500, len_hi=3000, top_k=256,
                        with_kv=False)
    case = synth.make_case(spec, seed)
    g = synth.rng(seed, "int_case")
    keys = g.integers(-4, 5, size=case.idx_keys.shape).astype(np.float32)
    case.idx_keys[...] = synth.to_bf16_bits(keys)
    case.q_idx[...] = synth.to_bf16_bits(g.integers(-2, 3, size=case.q_idx.shape).astype(np.float32))
    case.w[...] = g.integers(-2, 3, size=case.w.shape).astype(np.float32)
    bits = synth.to_e4m3_bits(keys)
    scales = np.ones(keys.shape[:-1], np.float32)
    return case, bits, scales


@pytest.mark.parametrize("n_cand", [256, 300, 1024, 4096])
def test_two_stage_bit_exact_on_integer_data(n_cand):
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case, bits, scales = _int_case(61)
    dc = DeviceCase(case)
    k = case.spec.top_k
    idx = torch.full((dc.rows, k), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.two_stage_workspace_size(dc.dims, dc.rows, dc.max_len, n_cand))
    lsa.two_stage_select(dc.dims, dc.cache, torch.from_numpy(bits).cuda(), torch.from_numpy(scales).cuda(),
                         dc.q_idx, dc.w, n_cand, idx, ws)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    got = idx.cpu().numpy()
    for r in range(dc.rows):
        want = O.two_stage_select(case, bits, scales, r, k, n_cand)
        assert np.array_equal(got[r], want), f"row {r}"
        if n_cand >= O.row_visible(case, r):
            assert np.array_equal(got[r], O.topk(O.row_scores(case, r), O.row_visible(case, r), k))


def _check_two_stage(got, want, compact, exact, L, n_cand, what):
    """Equal sizes, ascending, -1 padded; every position in the symmetric
    difference is a near tie of the oracle at the list's cut (compact score,
    FP8 score tolerance) or at the final cut (exact score, selection window)."""
    g = set(int(x) for x in got if x >= 0)
    w = set(int(x) for x in want if x >= 0)
    assert len(g) == len(w), f"{what}: sizes {len(g)} vs {len(w)}"
    n = len(g)
    assert (np.diff(got[:n]) > 0).all() and (got[n:] == -1).all(), f"{what}: order or padding"
    if not (g ^ w):
        return 0
    cut_c = np.sort(compact[:L])[::-1][min(n_cand, L) - 1]
    floor_c = 1e-2 * np.abs(compact[:L]).max()
    kth = exact[sorted(w)].min()
    for s in g ^ w:
        near_final = abs(exact[s] - kth) <= SEL_TOL * abs(kth)
        near_list = abs(compact[s] - cut_c) <= SCORE_TOL["fp8"] * max(abs(cut_c), floor_c)
        assert near_final or near_list, f"{what}: position {s} differs away from both cuts"
    return len(g ^ w)


@pytest.mark.parametrize("name,n_cand", [("paged_B5", 1024), ("bf16_L5000", 2048), ("prefill_3000x256", 1024)])
def test_two_stage_vs_oracle(name, n_cand):
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small(name)
    dc = DeviceCase(case)
    bits, scales, d_bits, d_scales = _compact_device(case)
    k = case.spec.top_k
    idx = torch.full((dc.rows, k), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.two_stage_workspace_size(dc.dims, dc.rows, dc.max_len, n_cand))
    lsa.two_stage_select(dc.dims, dc.cache, d_bits, d_scales, dc.q_idx, dc.w, n_cand, idx, ws,
                         row_seq=dc.row_seq, row_pos=dc.row_pos)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    got = idx.cpu().numpy()
    rows = range(dc.rows) if dc.rows <= 8 else [0, 1, 77, dc.rows - 1]
    for r in rows:
        L = O.row_visible(case, r)
        want = O.two_stage_select(case, bits, scales, r, k, n_cand)
        _check_two_stage(got[r], want, O.compact_row_scores(case, bits, scales, r), O.row_scores(case, r), L,
                         n_cand, f"{name} row {r}")


def test_two_stage_rejects_a_short_list():
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small("paged_B5")
    dc = DeviceCase(case)
    _, _, d_bits, d_scales = _compact_device(case)
    k = case.spec.top_k
    idx = torch.empty((dc.rows, k), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(1 << 20)
    assert lsa.two_stage_select(dc.dims, dc.cache, d_bits, d_scales, dc.q_idx, dc.w, k - 1, idx, ws,
                                raise_on_error=False) == lsa.LSA_ERR_INVALID_ARG
    assert lsa.two_stage_workspace_size(dc.dims, dc.rows, dc.max_len, k - 1) == 0


@pytest.mark.slow
def test_two_stage_full_batch():
    """The paged batch workload (B=32, 64K-128K tokens, k = 2048) with a list of
    8192, checked on sampled rows."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.full(synth.DECODE_B32, with_kv=False)
    dc = DeviceCase(case)
    bits, scales, d_bits, d_scales = _compact_device(case)
    k, n_cand = case.spec.top_k, 8192
    idx = torch.full((dc.rows, k), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.two_stage_workspace_size(dc.dims, dc.rows, dc.max_len, n_cand))
    lsa.two_stage_select(dc.dims, dc.cache, d_bits, d_scales, dc.q_idx, dc.w, n_cand, idx, ws)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    got = idx.cpu().numpy()
    for r in (0, dc.rows // 2, dc.rows - 1):
        L = O.row_visible(case, r)
        want = O.two_stage_select(case, bits, scales, r, k, n_cand)
        _check_two_stage(got[r], want, O.compact_row_scores(case, bits, scales, r), O.row_scores(case, r), L,
                         n_cand, f"B32 row {r}")
