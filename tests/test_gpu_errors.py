"""Error handling: host-side argument checks and device-side bounds checks.

Device errors are provoked only through inputs that the kernels' own bounds
checks catch (a block id outside the pool, a length above max_len, a selected
position past the sequence): the kernels skip the access, write NaN / skip the
row, and record the status word; nothing traps.
"""
import ctypes

import numpy as np
import pytest

from tests import cases

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _dc(name="paged_B5"):
    from sparse_attention_decode_scan_b200.device import DeviceCase
    return DeviceCase(cases.small(name))


def test_host_argument_errors():
    from sparse_attention_decode_scan_b200 import lsa
    dc = _dc()
    R = dc.rows
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((R, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, R, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    bad = lsa.Dims.from_buffer_copy(dc.dims)
    bad.n_idx_heads = 0
    assert lsa.indexer_scores(bad, dc.cache, dc.q_idx, dc.w, scores, ld, ws, raise_on_error=False) \
        == lsa.LSA_ERR_INVALID_ARG
    assert lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, dc.max_len - 1, ws,
                              raise_on_error=False) == lsa.LSA_ERR_INVALID_ARG
    small_ws = ws[:256]
    assert lsa.topk(scores, 16, torch.empty((R, 16), dtype=torch.int32, device="cuda"), small_ws,
                    raise_on_error=False) == lsa.LSA_ERR_WORKSPACE
    assert lsa.topk(scores, 16, torch.empty((R, 16), dtype=torch.int32, device="cuda"), ws[1:],
                    raise_on_error=False) == lsa.LSA_ERR_WORKSPACE
    assert lsa.topk(scores, 0, torch.empty((R, 1), dtype=torch.int32, device="cuda"), ws,
                    raise_on_error=False) == lsa.LSA_ERR_INVALID_ARG
    c = lsa.Cache.from_buffer_copy(dc.cache)
    c.kv = None
    out = torch.empty((R, dc.spec.n_heads, dc.spec.v_dim), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros((R, dc.spec.top_k), dtype=torch.int32, device="cuda")
    assert lsa.sparse_attn_decode(dc.dims, c, dc.q, idx, out, None, ws, raise_on_error=False) \
        == lsa.LSA_ERR_INVALID_ARG
    assert lsa.decode_step(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, out, None, ws, flags=7,
                           raise_on_error=False) == lsa.LSA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK


@pytest.mark.parametrize("path", ["default", "simt"])
def test_block_id_out_of_pool_is_reported(path, request):
    if path == "simt":
        request.getfixturevalue("test_hooks")(force_simt=True)
    from sparse_attention_decode_scan_b200 import lsa
    dc = _dc()
    bt = dc.block_table.clone()
    bt[1, 0] = int(dc.cache.n_blocks) + 5      # outside the pool
    dc.block_table = bt
    dc.cache = dc.make_cache()
    R = dc.rows
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.zeros((R, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, R, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_ERR_BOUNDS
    s = scores.cpu().numpy()
    bs = dc.spec.block_size
    assert np.isnan(s[1, :bs]).all() and np.isfinite(s[0, :int(dc.case.seq_lens[0])]).all()
    # the context stays usable and the status word was cleared
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_ERR_BOUNDS
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    # the single-status form reads and clears the same word
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq)
    assert lsa.get_device_status(ws) == lsa.LSA_ERR_BOUNDS
    assert lsa.get_device_status(ws) == lsa.LSA_OK


def test_length_above_max_len_is_reported():
    from sparse_attention_decode_scan_b200 import lsa
    dc = _dc("bf16_L5000")
    dc.seq_lens = torch.tensor([dc.max_len + 100], dtype=torch.int32, device="cuda")
    dc.cache = dc.make_cache()
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.zeros((1, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, 1, dc.max_len, lsa.LSA_OP_SCORES))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_ERR_BOUNDS
    assert np.isfinite(scores.cpu().numpy()[0, :dc.max_len]).all()


def test_selected_position_past_length_is_reported():
    from sparse_attention_decode_scan_b200 import lsa
    dc = _dc()
    R, k = dc.rows, dc.spec.top_k
    idx = torch.full((R, k), -1, dtype=torch.int32, device="cuda")
    idx[0, 0] = int(dc.case.seq_lens[0]) + 3
    idx[0, 1] = 0
    out = torch.empty((R, dc.spec.n_heads, dc.spec.v_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((R, dc.spec.n_heads), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, R, dc.max_len, lsa.LSA_OP_ATTN))
    lsa.sparse_attn_decode(dc.dims, dc.cache, dc.q, idx, out, lse, ws)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_ERR_BOUNDS
    assert np.isfinite(out.float().cpu().numpy()[0]).all()
