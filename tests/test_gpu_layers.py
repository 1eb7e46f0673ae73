"""Several DSA layers of one decode step through lsa_decode_layers (IndexCache
and Multi-layer Indexer routes) against the oracle, and against the
single-layer entry points composed by hand."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests.helpers import check_attention, check_selection

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _spec(**kw):
    # production widths (tensor-core scan and attention), paged, ragged lengths
    base = dict(batch=3, len_lo=300, len_hi=2500, top_k=256)
    base.update(kw)
    return synth.scaled(synth.WORKLOADS[synth.DECODE_B32], **base)


def _run_layers(dls, retention, route):
    from sparse_attention_decode_scan_b200 import lsa
    s = dls[0].spec
    B, n = dls[0].rows, len(dls)
    outs = [torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda") for _ in dls]
    lses = [torch.empty((B, s.n_heads), dtype=torch.float32, device="cuda") for _ in dls]
    idx = torch.full((n, B, s.top_k), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dls[0].dims, B, dls[0].max_len, lsa.LSA_OP_DECODE_LAYERS))
    lsa.decode_layers(dls[0].dims, [d.cache for d in dls], [d.q_idx for d in dls], [d.w for d in dls],
                      [d.q for d in dls], outs, lses, ws, retention=retention, route=route, idx_out=idx)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    return [o.float().cpu().numpy() for o in outs], [x.cpu().numpy() for x in lses], idx.cpu().numpy()


@pytest.mark.parametrize("retention", [1, 2])
@pytest.mark.parametrize("route", [O.ROUTE_OWN, O.ROUTE_PREV])
def test_layers_match_the_oracle(retention, route):
    from sparse_attention_decode_scan_b200.device import device_layers
    layers = synth.make_layers(_spec(), 8101, 4)
    dls = device_layers(layers)
    out, lse, idx = _run_layers(dls, retention, route)
    src, ref = O.decode_layers(layers, retention, route)
    for l in range(len(layers)):
        ref_idx, o_ref, l_ref = ref[l]
        for r in range(layers[l].rows):
            what = f"layer {l} (selection of layer {src[l]}) row {r}"
            sc = O.row_scores(layers[src[l]], r)
            check_selection(idx[l, r], ref_idx[r], sc, what=what)
            if np.array_equal(idx[l, r], ref_idx[r]):
                check_attention(out[l][r], o_ref[r], lse[l][r], l_ref[r], what=what)


def _single(dc, idx=None):
    """One layer through the single-layer entry points: its own step, or its
    attention on a given selection."""
    from sparse_attention_decode_scan_b200 import lsa
    s = dc.spec
    B = dc.rows
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device="cuda")
    if idx is None:
        idx = torch.empty((B, s.top_k), dtype=torch.int32, device="cuda")
        ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
        lsa.decode_step(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, out, lse, ws, idx_out=idx)
    else:
        ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_ATTN))
        lsa.sparse_attn_decode(dc.dims, dc.cache, dc.q, idx, out, lse, ws, row_seq=dc.row_seq)
    torch.cuda.synchronize()
    return out, lse, idx


@pytest.mark.parametrize("shape", ["small", "long_B4"])
def test_mli_layers_equal_the_composed_single_layer_calls(shape):
    """Under the MLI route layer l's output is, bit for bit, the attention of
    layer l on layer l-1's own selection (retention 1)."""
    from sparse_attention_decode_scan_b200.device import device_layers
    spec = _spec() if shape == "small" else _spec(batch=4, len_lo=65536, len_hi=131072, top_k=2048)
    layers = synth.make_layers(spec, 8102, 3)
    dls = device_layers(layers)
    out, lse, idx = _run_layers(dls, 1, O.ROUTE_PREV)
    own = [_single(d) for d in dls]
    for l, d in enumerate(dls):
        src = max(l - 1, 0)
        assert np.array_equal(idx[l], own[src][2].cpu().numpy()), f"layer {l} selection"
        o, ls, _ = own[0] if l == 0 else _single(d, own[src][2])
        assert np.array_equal(out[l], o.float().cpu().numpy()), f"layer {l} output"
        assert np.array_equal(lse[l], ls.cpu().numpy()), f"layer {l} lse"


def test_identical_layers_make_the_routes_agree_on_the_gpu():
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(synth.make_case(_spec(), 8103))
    a = _run_layers([dc] * 3, 1, O.ROUTE_OWN)
    b = _run_layers([dc] * 3, 1, O.ROUTE_PREV)
    for x, y in zip(a, b):
        for u, v in zip(x, y):
            assert np.array_equal(u, v)


def test_layer_arguments_are_checked_before_any_launch():
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase, device_layers
    layers = synth.make_layers(_spec(batch=2, len_lo=200, len_hi=300), 8104, 2)
    dls = device_layers(layers)
    s = dls[0].spec
    outs = [torch.empty((2, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda") for _ in dls]
    ws = lsa.workspace(lsa.workspace_size(dls[0].dims, 2, dls[0].max_len, lsa.LSA_OP_DECODE_LAYERS))

    def call(dl, retention=1, route=lsa.LSA_ROUTE_PREV, wsz=ws):
        return lsa.decode_layers(dls[0].dims, [d.cache for d in dl], [d.q_idx for d in dl], [d.w for d in dl],
                                 [d.q for d in dl], outs[:len(dl)], None, wsz, retention=retention, route=route,
                                 raise_on_error=False)

    assert call(dls, retention=0) == lsa.LSA_ERR_INVALID_ARG
    assert call(dls, route=7) == lsa.LSA_ERR_INVALID_ARG
    # a layer with its own copy of the lengths (not the batch's shared array)
    other = DeviceCase(layers[1])
    assert call([dls[0], other]) == lsa.LSA_ERR_INVALID_ARG
    assert call(dls, wsz=ws[:1024]) == lsa.LSA_ERR_WORKSPACE
    assert call(dls) == lsa.LSA_OK
    torch.cuda.synchronize()
