"""lsa_topk_noalloc against lsa_topk, through the C ABI.

lsa_topk_noalloc serves callers that cannot allocate device memory where they
call the top-k (plugin hosts that forbid allocation on their enqueue path,
runtimes whose memory is all pre-reserved, latency-critical loops).  Its scratch
is a static array inside the library, shared by every call, so two calls in a
row must both match the workspace entry point exactly (the top-k tolerance is
bit-exact).  This file is collected last on purpose.
"""
import numpy as np
import pytest

from sparse_attention_decode_scan_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def _both(sc: np.ndarray, k: int, valid=None):
    from sparse_attention_decode_scan_b200 import lsa
    rows, n = sc.shape
    dev = torch.from_numpy(sc).cuda()
    vdev = torch.from_numpy(valid).cuda() if valid is not None else None
    ref = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.topk_workspace_size(rows, n, k))
    lsa.topk(dev, k, ref, ws, valid_len=vdev)
    got = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    lsa.topk_noalloc(dev, k, got, valid_len=vdev)
    torch.cuda.synchronize()
    return ref.cpu().numpy(), got.cpu().numpy()


def test_noalloc_matches_workspace_topk_twice():
    # first call: 32 rows of ragged 128K-scale rows; second: different rows, ties
    sc1 = synth.topk_scores("normal", 32, 131072, 71)
    valid = np.random.default_rng(72).integers(65536, 131073, 32).astype(np.int32)
    ref1, got1 = _both(sc1, 2048, valid)
    assert np.array_equal(ref1, got1)
    sc2 = synth.topk_scores("ties", 5, 40000, 73)
    ref2, got2 = _both(sc2, 777)
    assert np.array_equal(ref2, got2)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    from sparse_attention_decode_scan_b200 import lsa
    rows, n = 200, 4096  # 200 rows of top-k scratch exceed the 4 MiB array
    dev = torch.zeros((rows, n), dtype=torch.float32, device="cuda")
    idx = torch.empty((rows, 8), dtype=torch.int32, device="cuda")
    assert lsa.topk_noalloc(dev, 8, idx, raise_on_error=False) == lsa.LSA_ERR_UNSUPPORTED
