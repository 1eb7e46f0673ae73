"""Block-level selection and the staged copy of the kept blocks (SparDA
abstract, page 4 of the sources) against the oracle's block_select and its
attention over the kept blocks' positions."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests import cases
from tests.helpers import SEL_TOL, check_attention

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("kind,rows,n,bs,n_sel,ragged", [
    ("normal", 3, 5000, 64, 8, False), ("ties", 4, 10000, 64, 20, True), ("heavy", 2, 131072, 64, 32, True),
    ("equal", 2, 3000, 7, 5, False), ("signed_zero_inf", 3, 7000, 16, 40, True), ("normal", 2, 100, 64, 4, False)])
def test_block_select_exact(kind, rows, n, bs, n_sel, ragged):
    """Fixed fp32 scores: the kept blocks equal the oracle's bit for bit."""
    from sparse_attention_decode_scan_b200 import lsa
    seed = 300 + n % 101 + bs
    sc = synth.topk_scores(kind, rows, n, seed)
    valid = np.random.default_rng(seed).integers(n // 2, n + 1, rows).astype(np.int32) if ragged else None
    ld = (n + 3) // 4 * 4
    dev = torch.full((rows, ld), float("nan"), dtype=torch.float32, device="cuda")
    dev[:, :n] = torch.from_numpy(sc).cuda()
    kept = torch.full((rows, n_sel), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.block_select_workspace_size(rows, n, bs, n_sel))
    lsa.block_select(dev, bs, n_sel, kept, ws, valid_len=torch.from_numpy(valid).cuda() if ragged else None,
                     n_cols=n, ld=ld)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    got = kept.cpu().numpy()
    for r in range(rows):
        L = n if valid is None else int(valid[r])
        assert np.array_equal(got[r], O.block_select(sc[r].astype(np.float32), L, bs, n_sel)), f"row {r}"


def _stage_and_attend(lsa, dc, kept_np, bs, kv_ptr=None):
    s = dc.spec
    R, n_sel = dc.rows, kept_np.shape[1]
    kept = torch.from_numpy(np.ascontiguousarray(kept_np)).cuda()
    odt = torch.float32 if s.act_dtype == "f32" else torch.bfloat16
    staged = torch.empty((R * n_sel, bs, s.qk_dim), dtype=odt, device="cuda")
    table = torch.empty((R, n_sel), dtype=torch.int32, device="cuda")
    sidx = torch.empty((R, n_sel * bs), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(256)
    cache = dc.make_cache()
    if kv_ptr is not None:
        cache.kv = kv_ptr
    lsa.stage_blocks(dc.dims, cache, kept, bs, staged, table, sidx, ws, row_seq=dc.row_seq, row_pos=dc.row_pos)
    lens = torch.full((R,), n_sel * bs, dtype=torch.int32, device="cuda")
    sc = lsa.staged_cache(staged, table, lens, n_sel, bs)
    from sparse_attention_decode_scan_b200.device import make_dims
    d = make_dims(s, top_k=n_sel * bs)
    d.block_size = bs
    out = torch.empty((R, s.n_heads, s.v_dim), dtype=odt, device="cuda")
    lse = torch.empty((R, s.n_heads), dtype=torch.float32, device="cuda")
    ws2 = lsa.workspace(lsa.workspace_size(d, R, n_sel * bs, lsa.LSA_OP_ATTN))
    lsa.sparse_attn_decode(d, sc, dc.q, sidx, out, lse, ws2)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK and lsa.read_device_status(ws2) == lsa.LSA_OK
    return staged, out.float().cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("name,n_sel", [("paged_B5", 8), ("bf16_L5000", 32), ("tiny_fp32", 4),
                                        ("prefill_3000x256", 8)])
def test_block_selection_and_staged_attention_vs_oracle(name, n_sel):
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small(name)
    dc = DeviceCase(case)
    s = case.spec
    bs = s.block_size or 64
    R = dc.rows
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((R, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(max(lsa.workspace_size(dc.dims, R, dc.max_len, lsa.LSA_OP_SCORES),
                           lsa.block_select_workspace_size(R, dc.max_len, bs, n_sel)))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq, row_pos=dc.row_pos)
    kept = torch.empty((R, n_sel), dtype=torch.int32, device="cuda")
    lsa.block_select(scores, bs, n_sel, kept, ws, n_cols=dc.max_len, ld=ld)
    torch.cuda.synchronize()
    got = kept.cpu().numpy()
    rows = range(R) if R <= 8 else [0, 1, 77, R - 1]
    ref = np.full((R, n_sel), -1, np.int32)
    for r in rows:
        L = O.row_visible(case, r)
        bsc = O.block_scores(O.row_scores(case, r), L, bs)
        ref[r] = O.block_select(O.row_scores(case, r), L, bs, n_sel)
        g, w = set(got[r][got[r] >= 0].tolist()), set(ref[r][ref[r] >= 0].tolist())
        assert len(g) == len(w)
        if g ^ w:
            kth = bsc[sorted(w)].min()
            for blk in g ^ w:
                assert abs(bsc[blk] - kth) <= SEL_TOL * abs(kth), f"{name} row {r}: block {blk} outside the tie window"
    # the staged copy and the attention over it, on the oracle's kept blocks
    _, o, l = _stage_and_attend(lsa, dc, ref, bs)
    for r in rows:
        _, pos, o_ref, l_ref = O.row_block_step(case, r, n_sel, block_size=bs)
        check_attention(o[r], o_ref, l[r], l_ref, what=f"{name} row {r}")


def test_staging_from_host_memory_equals_device():
    """An offloaded KV cache: the same staged blocks read from page-locked host memory."""
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small("paged_B5")
    dc = DeviceCase(case)
    n_sel, bs = 8, case.spec.block_size
    kept = np.stack([O.block_select(O.row_scores(case, r), O.row_visible(case, r), bs, n_sel)
                     for r in range(dc.rows)])
    dev_staged, o1, l1 = _stage_and_attend(lsa, dc, kept, bs)
    host_kv = dc.kv.cpu().pin_memory()
    host_staged, o2, l2 = _stage_and_attend(lsa, dc, kept, bs, kv_ptr=host_kv.data_ptr())
    assert torch.equal(dev_staged, host_staged)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_stage_blocks_rejects_unusable_arguments():
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = cases.small("paged_B5")
    dc = DeviceCase(case)
    R, n_sel = dc.rows, 4
    kept = torch.zeros((R, n_sel), dtype=torch.int32, device="cuda")
    staged = torch.empty((R * n_sel, 64, 576), dtype=torch.bfloat16, device="cuda")
    table = torch.empty((R, n_sel), dtype=torch.int32, device="cuda")
    sidx = torch.empty((R, n_sel * 64), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(256)
    # a paged cache's blocks are its pages
    assert lsa.stage_blocks(dc.dims, dc.cache, kept, 32, staged, table, sidx, ws,
                            raise_on_error=False) == lsa.LSA_ERR_INVALID_ARG
    # host memory the device cannot map
    plain = np.zeros(1 << 20, np.uint8)
    c = dc.make_cache()
    c.kv = plain.ctypes.data
    assert lsa.stage_blocks(dc.dims, c, kept, 64, staged, table, sidx, ws,
                            raise_on_error=False) == lsa.LSA_ERR_INVALID_ARG
