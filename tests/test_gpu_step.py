"""End-to-end decode step (scan -> top-k -> sparse MQA) and the prefill chain vs the oracle."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests import cases
from tests.helpers import check_attention, check_selection

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _step(dc, flags=0):
    from sparse_attention_decode_scan_b200 import lsa
    s = dc.spec
    B = dc.rows
    odt = torch.float32 if s.act_dtype == "f32" else torch.bfloat16
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=odt, device="cuda")
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, s.top_k), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    lsa.decode_step(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, out, lse, ws, idx_out=idx, flags=flags)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    return out, lse, idx


def _attn_on(dc, idx_np):
    from sparse_attention_decode_scan_b200 import lsa
    s = dc.spec
    B = dc.rows
    odt = torch.float32 if s.act_dtype == "f32" else torch.bfloat16
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=odt, device="cuda")
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_ATTN))
    lsa.sparse_attn_decode(dc.dims, dc.cache, dc.q, torch.from_numpy(idx_np).cuda(), out, lse, ws,
                           row_seq=dc.row_seq)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def _check_step(case, rows, flags=0):
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(case)
    out, lse, idx = _step(dc, flags)
    out_h, lse_h, idx_h = out.float().cpu().numpy(), lse.cpu().numpy(), idx.cpu().numpy()
    ref_sel = np.stack([O.topk(O.row_scores(case, r), O.row_visible(case, r), case.spec.top_k)
                        if r in rows else np.full(case.spec.top_k, -1, np.int32) for r in range(case.rows)])
    # GPU attention on the oracle's selection (same selection on both sides)
    o_gpu_on_ref, l_gpu_on_ref = _attn_on(dc, ref_sel)
    ndiff = 0
    for r in rows:
        sc = O.row_scores(case, r)
        ndiff += check_selection(idx_h[r], ref_sel[r], sc, what=f"{case.spec.name} row {r}")
        o_ref, l_ref = O.row_attention(case, r, ref_sel[r])
        check_attention(o_gpu_on_ref[r], o_ref, l_gpu_on_ref[r], l_ref, what=f"{case.spec.name} row {r}")
        if np.array_equal(idx_h[r], ref_sel[r]):
            check_attention(out_h[r], o_ref, lse_h[r], l_ref, what=f"{case.spec.name} step row {r}")
    return ndiff


@pytest.mark.parametrize("name", ["tiny_fp32", "bf16_L5000", "paged_B5", "fp8_L6001", "len1"])
def test_decode_step_small(name):
    case = cases.small(name)
    _check_step(case, list(range(case.rows)))


@pytest.mark.parametrize("name", ["tiny_fp32", "bf16_L5000", "paged_B5", "fp8_L6001", "len1"])
def test_decode_step_fused_bitwise_equals_unfused(name):
    """The fused step runs the CTA code of the separate launches with the same
    plans, so selection, output and lse agree bit for bit (tiny_fp32 takes the
    separate CUDA-core launches under either flag)."""
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(cases.small(name))
    o1, l1, i1 = _step(dc, 0)
    o2, l2, i2 = _step(dc, 1)
    assert torch.equal(i1, i2)
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


@pytest.mark.parametrize("name", ["bf16_L5000", "paged_B5", "fp8_L6001", "len1"])
def test_decode_step_fused_vs_oracle(name):
    case = cases.small(name)
    _check_step(case, list(range(case.rows)), flags=1)


def _phase_ms(dc, flags):
    from sparse_attention_decode_scan_b200 import lsa
    s = dc.spec
    B = dc.rows
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
    for e in ev:  # torch creates (and marks recorded) an event at its first record
        e.record()
    for _ in range(2):
        lsa.decode_step_profiled(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, out, lse, ws, ev, flags=flags)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    return [ev[i].elapsed_time(ev[i + 1]) for i in range(3)]


@pytest.mark.parametrize("name", ["paged_B5", "fp8_L6001"])
def test_fused_step_is_one_launch(name):
    """With LSA_STEP_FUSED the whole step is the one launch between the first
    two phase events (the later events follow it immediately)."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(cases.small(name))
    assert lsa.launch_count(dc.dims, dc.rows, dc.max_len, lsa.LSA_OP_DECODE_STEP_FUSED) == 1
    assert lsa.launch_count(dc.dims, dc.rows, dc.max_len, lsa.LSA_OP_DECODE_STEP) >= 3
    fused = _phase_ms(dc, 1)
    unfused = _phase_ms(dc, 0)
    assert fused[0] > 0.0
    assert fused[1] < 0.01 and fused[2] < 0.01, fused      # nothing runs after the single launch
    assert unfused[1] > 0.002 and unfused[2] > 0.002, unfused  # top-k and attention launches


def test_prefill_chain_small():
    """Causal scores -> top-k over every row -> attention over each row's selection."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small("prefill_3000x256")
    dc = DeviceCase(case)
    R, k = dc.rows, case.spec.top_k
    L = int(case.seq_lens[0])
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((R, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(max(lsa.workspace_size(dc.dims, R, dc.max_len, op) for op in range(3)))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq, row_pos=dc.row_pos)
    idx = torch.empty((R, k), dtype=torch.int32, device="cuda")
    lsa.topk(scores, k, idx, ws, n_cols=L, ld=ld)
    torch.cuda.synchronize()
    idx_h = idx.cpu().numpy()
    for r in [0, 1, 77, R - 1]:
        sc = O.row_scores(case, r)
        ref = O.topk(sc, L, k)
        check_selection(idx_h[r], ref, sc, what=f"prefill row {r}")
        assert (idx_h[r][idx_h[r] >= 0] <= case.row_pos[r]).all()


@pytest.mark.slow
def test_prefill_chain_full():
    """The full prefill workload (8192 chunk rows at positions 131072..139263
    over 139264 tokens, causal): lsa_indexer_scores with the rows' positions,
    lsa_topk over every row, lsa_sparse_attn_decode for every row, in the
    launch configuration the benchmark times.  Checked on sampled rows (first,
    last and random): the selection against the oracle's top-k of the oracle's
    scores, and the attention run on the oracle's selection against the
    oracle's attention."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.full(synth.PREFILL)
    dc = DeviceCase(case)
    R, k = dc.rows, case.spec.top_k
    L = int(case.seq_lens[0])
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((R, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(max(lsa.workspace_size(dc.dims, R, dc.max_len, op) for op in range(3)))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq, row_pos=dc.row_pos)
    idx = torch.empty((R, k), dtype=torch.int32, device="cuda")
    lsa.topk(scores, k, idx, ws, n_cols=L, ld=ld)
    out = torch.empty((R, case.spec.n_heads, case.spec.v_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((R, case.spec.n_heads), dtype=torch.float32, device="cuda")
    lsa.sparse_attn_decode(dc.dims, dc.cache, dc.q, idx, out, lse, ws, row_seq=dc.row_seq)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    idx_h = idx.cpu().numpy()
    out_h = out.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    g = np.random.default_rng(8192)
    rows = sorted({0, 1, R - 1, *g.integers(2, R - 1, 5).tolist()})
    ref_sel = np.full((R, k), -1, np.int32)
    for r in rows:
        sc = O.row_scores(case, r)
        ref_sel[r] = O.topk(sc, L, k)
        check_selection(idx_h[r], ref_sel[r], sc, what=f"prefill row {r}")
        assert (idx_h[r][idx_h[r] >= 0] <= case.row_pos[r]).all()
    o_on_ref, l_on_ref = _attn_on(dc, ref_sel)
    for r in rows:
        o_ref, l_ref = O.row_attention(case, r, ref_sel[r])
        check_attention(o_on_ref[r], o_ref, l_on_ref[r], l_ref, what=f"prefill attention row {r}")
        if np.array_equal(idx_h[r], ref_sel[r]):
            check_attention(out_h[r], o_ref, lse_h[r], l_ref, what=f"prefill chain row {r}")


@pytest.mark.slow
@pytest.mark.parametrize("name", [synth.DECODE_B1, synth.DECODE_B32])
def test_decode_step_full(name):
    case = cases.full(name)
    rows = sorted({0, case.rows - 1, case.rows // 2})
    _check_step(case, rows)


@pytest.mark.slow
def test_decode_step_full_fp8():
    case = cases.full(synth.DECODE_B4_FP8)
    _check_step(case, [0, 3])


@pytest.mark.slow
@pytest.mark.parametrize("name", [synth.DECODE_B1, synth.DECODE_B32, synth.DECODE_B4_FP8])
def test_decode_step_full_fused_bitwise_equals_unfused(name):
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(cases.full(name))
    o1, l1, i1 = _step(dc, 0)
    o2, l2, i2 = _step(dc, 1)
    assert torch.equal(i1, i2)
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)


@pytest.mark.slow
def test_decode_step_full_fused_vs_oracle():
    case = cases.full(synth.DECODE_B32)
    rows = sorted({0, case.rows - 1, case.rows // 2})
    _check_step(case, rows, flags=1)


@pytest.mark.parametrize("name", ["paged_B5", "fp8_L6001", "bf16_L5000"])
def test_decode_step_selection_equals_separate_calls(name):
    """lsa_decode_step (whose scan may also build the top-k's first histogram)
    selects exactly what lsa_indexer_scores followed by lsa_topk selects."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(cases.small(name))
    _, _, idx_step = _step(dc)
    B, k = dc.rows, dc.spec.top_k
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((B, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    lsa.topk(scores, k, idx, ws, valid_len=dc.seq_lens, n_cols=dc.max_len, ld=ld)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_step)


def _split_case():
    """Decode case for the split select: 4 sequences of 5000-6000 tokens (k = 512)
    where sequence 0 is cut to 200 tokens whose keys are all one key (every
    score equal: 200 ties at the threshold, ranked by the split select itself)
    and sequence 1 keeps its length with all keys equal too (more ties than the
    split select ranks: the row falls back to the full select)."""
    from sparse_attention_decode_scan_b200 import synth
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=4, len_lo=5000, len_hi=6000, top_k=512)
    case = synth.make_case(spec, 7101)
    bs = spec.block_size
    case.seq_lens[0] = 200
    for b in (0, 1):
        first = case.block_table[b][0]
        key = case.idx_keys[first, 0].copy()
        for p in range(int(case.seq_lens[b])):
            case.idx_keys[case.block_table[b][p // bs], p % bs] = key
    return case


@pytest.mark.parametrize("min_cols,no_cluster", [(0, True), (100000000, True), (100000000, False)])
def test_decode_step_split_select(min_cols, no_cluster, test_hooks):
    """With the split select forced on (rows of any length; the cluster top-k,
    which rows that short would otherwise take, turned off) or off (the
    collect + select or the cluster top-k), the decode step selects what
    lsa_indexer_scores + lsa_topk select, ties and the fallback row included,
    and its outputs match the oracle."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    test_hooks(split_select_min_cols=min_cols, no_cluster_topk=no_cluster)
    case = _split_case()
    dc = DeviceCase(case)
    _, _, idx_step = _step(dc)
    B, k = dc.rows, dc.spec.top_k
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((B, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws)
    idx = torch.empty((B, k), dtype=torch.int32, device="cuda")
    lsa.topk(scores, k, idx, ws, valid_len=dc.seq_lens, n_cols=dc.max_len, ld=ld)
    torch.cuda.synchronize()
    assert torch.equal(idx, idx_step)
    # all-equal rows keep the lowest positions
    assert (idx_step[0, :200].cpu().numpy() == np.arange(200)).all() and (idx_step[0, 200:] == -1).all()
    assert (idx_step[1].cpu().numpy() == np.arange(k)).all()
    _check_step(case, list(range(B)))
    # unfused and fused agree bit for bit (the fused step never splits)
    o1, l1, i1 = _step(dc, 0)
    o2, l2, i2 = _step(dc, 1)
    assert torch.equal(i1, i2) and torch.equal(o1, o2) and torch.equal(l1, l2)
