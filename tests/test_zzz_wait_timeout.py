"""A decode-step wait that runs out: the step's top-k waits for a count of scan
CTAs that is never reached (the scan_wait_extra switch of the test build,
liblsa_test.so), so its bounded wait and
then the attention's wait on the rows' selection flags give up after their
limit (about a second each).  The status word must hold LSA_ERR_TIMEOUT, and
the same context must then run an ordinary step cleanly.  Nothing faults or
traps.  Collected last on purpose (it takes a few seconds)."""
import numpy as np
import pytest

from tests import cases

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_step_wait_times_out_and_the_context_recovers(test_hooks):
    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase
    dc = DeviceCase(cases.small("bf16_L5000"))
    s = dc.spec
    B = dc.rows
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device="cuda")
    idx = torch.empty((B, s.top_k), dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    # the handoff this hook breaks exists with the tensor-core scan and the one-launch top-k
    assert lsa.launch_count(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP) == 3
    test_hooks(scan_wait_extra=1)
    lsa.decode_step(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_ERR_TIMEOUT
    test_hooks(scan_wait_extra=0)
    # the same context, workspace and buffers: an ordinary step is clean
    lsa.decode_step(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, out, lse, ws, idx_out=idx)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    ref = torch.empty_like(out)
    ws2 = lsa.workspace(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_DECODE_STEP))
    lsa.decode_step(dc.dims, dc.cache, dc.q_idx, dc.w, dc.q, ref, None, ws2)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert np.isfinite(lse.cpu().numpy()).all()
