"""Prefill through several layers with each layer's history streamed through two
alternating device buffers (LeanSparse episode page, summary), against the same
kernels on each layer's whole device-resident cache and against the oracle."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests import cases
from tests.helpers import check_attention, check_selection

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _layers(n_layers):
    from sparse_attention_decode_scan_b200.device import device_layers
    spec = cases.SMALL["prefill_3000x256"]
    layers = synth.make_layers(spec, 4321, n_layers)
    return layers, device_layers(layers)


def _reference(dc):
    """The unstreamed path on the layer's whole device cache."""
    from sparse_attention_decode_scan_b200 import lsa
    s = dc.spec
    R = dc.rows
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((R, ld), dtype=torch.float32, device="cuda")
    ws = lsa.workspace(max(lsa.workspace_size(dc.dims, R, dc.max_len, op) for op in range(3)))
    lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq, row_pos=dc.row_pos)
    idx = torch.empty((R, s.top_k), dtype=torch.int32, device="cuda")
    lsa.topk(scores, s.top_k, idx, ws, n_cols=dc.max_len, ld=ld)
    out = torch.empty((R, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((R, s.n_heads), dtype=torch.float32, device="cuda")
    lsa.sparse_attn_decode(dc.dims, dc.cache, dc.q, idx, out, lse, ws, row_seq=dc.row_seq)
    torch.cuda.synchronize()
    return out, lse, idx


def _streamed(dcs, row_block, host=True):
    from sparse_attention_decode_scan_b200 import lsa
    d0 = dcs[0]
    s = d0.spec
    R, L = d0.rows, d0.max_len
    hist_len = int(d0.case.row_pos[0])  # the chunk's own rows follow the history
    keep, caches, chunks = [], [], []
    for dc in dcs:
        hist = dc.kv[0, :hist_len]
        hist = hist.cpu().pin_memory() if host else hist.contiguous()
        chunk = dc.kv[0, hist_len:L].contiguous()
        keep += [hist, chunk]
        c = dc.make_cache()
        c.kv = hist.data_ptr()
        caches.append(c)
        chunks.append(chunk)
    outs = [torch.empty((R, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda") for _ in dcs]
    lses = [torch.empty((R, s.n_heads), dtype=torch.float32, device="cuda") for _ in dcs]
    idxs = [torch.empty((R, s.top_k), dtype=torch.int32, device="cuda") for _ in dcs]
    bufs = [torch.empty((L, s.qk_dim), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    ws = lsa.workspace(lsa.prefill_layers_workspace_size(d0.dims, R, L, row_block))
    events = [torch.cuda.Event() for _ in range(4)]
    copy = torch.cuda.Stream()
    lsa.prefill_layers(d0.dims, caches, hist_len, chunks, d0.row_pos, [dc.q_idx for dc in dcs], [dc.w for dc in dcs],
                       [dc.q for dc in dcs], outs, lses, bufs, ws, row_block, events, idx_out=idxs, copy_stream=copy)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    return outs, lses, idxs


@pytest.mark.parametrize("host", [True, False])
def test_streamed_layers_equal_the_resident_path_bitwise(host):
    """row_block >= rows: the same launches per layer as the whole-cache path."""
    layers, dcs = _layers(3)
    outs, lses, idxs = _streamed(dcs, row_block=1 << 20, host=host)
    for l, dc in enumerate(dcs):
        o, ls, ix = _reference(dc)
        assert torch.equal(idxs[l], ix), f"layer {l} selection"
        assert torch.equal(outs[l], o) and torch.equal(lses[l], ls), f"layer {l} output"


def test_streamed_layers_in_row_blocks_vs_oracle():
    """Rows in blocks of 100 (bounded score workspace): the selection equals the
    whole-cache path's exactly; outputs against the oracle on sampled rows."""
    layers, dcs = _layers(3)
    outs, lses, idxs = _streamed(dcs, row_block=100)
    for l, (case, dc) in enumerate(zip(layers, dcs)):
        _, _, ix = _reference(dc)
        assert torch.equal(idxs[l], ix), f"layer {l} selection"
        o_h, l_h, i_h = outs[l].float().cpu().numpy(), lses[l].cpu().numpy(), idxs[l].cpu().numpy()
        for r in (0, 99, 100, 255):
            sc = O.row_scores(case, r)
            ref = O.topk(sc, O.row_visible(case, r), case.spec.top_k)
            ndiff = check_selection(i_h[r], ref, sc, what=f"layer {l} row {r}")
            if ndiff == 0:  # same selection on both sides: the outputs must agree
                o_ref, lse_ref = O.row_attention(case, r, ref)
                check_attention(o_h[r], o_ref, l_h[r], lse_ref, what=f"layer {l} row {r}")
