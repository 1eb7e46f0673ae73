"""Top-k on fixed fp32 scores: bit-exact against the oracle."""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# (score kind, rows, n_cols, k, valid-length mode)
CASES = [
    ("normal", 1, 32768, 2048, "full"),        # single production row
    ("normal", 4, 524288, 2048, "full"),       # 4 x 512K
    ("normal", 32, 131072, 2048, "ragged"),    # batch of 32, lengths 64K..128K
    ("ties", 3, 10000, 500, "full"),
    ("equal", 2, 5000, 100, "full"),
    ("signed_zero_inf", 3, 7000, 3000, "full"),
    ("heavy", 2, 70000, 2048, "full"),
    ("neg", 2, 9000, 2048, "full"),
    ("normal", 3, 1000, 2048, "full"),         # k > n: -1 padding
    ("normal", 5, 4099, 1, "ragged"),
    ("normal", 1, 5, 3, "full"),
    ("normal", 4, 3000, 64, "with_zero"),      # a row with no valid entry
    ("ties", 40, 139264, 2048, "ragged"),      # many rows
    ("equal", 1, 200000, 2048, "full"),        # one tie class spread over many segments
    # 2^18 .. 2^19 positions: clusters of 16 CTAs (one overflowing every candidate list)
    ("ties", 2, 400000, 2048, "ragged"),
    ("equal", 1, 500000, 2048, "full"),
    # rows longer than 2^19 positions take the general five-launch path
    ("normal", 2, 600000, 2048, "full"),
    ("ties", 2, 600000, 2048, "ragged"),
    ("heavy", 1, 1 << 20, 4096, "full"),
]


def _valid(mode, rows, n, seed):
    g = np.random.default_rng(seed)
    if mode == "full":
        return None
    if mode == "ragged":
        return g.integers(max(1, n // 2), n + 1, rows).astype(np.int32)
    if mode == "with_zero":
        v = g.integers(1, n + 1, rows).astype(np.int32)
        v[1] = 0
        return v
    raise ValueError(mode)


@pytest.mark.parametrize("kind,rows,n,k,mode", CASES, ids=[f"{c[0]}-{c[1]}x{c[2]}-k{c[3]}-{c[4]}" for c in CASES])
def test_topk_exact(kind, rows, n, k, mode):
    from sparse_attention_decode_scan_b200 import lsa
    seed = 900 + rows + n % 97 + k
    sc = synth.topk_scores(kind, rows, n, seed)
    valid = _valid(mode, rows, n, seed)
    ld = (n + 3) // 4 * 4
    dev = torch.full((rows, ld), float("nan"), dtype=torch.float32, device="cuda")
    dev[:, :n] = torch.from_numpy(sc).cuda()
    vdev = torch.from_numpy(valid).cuda() if valid is not None else None
    idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
    ws = lsa.workspace(lsa.topk_workspace_size(rows, n, k))
    lsa.topk(dev, k, idx, ws, valid_len=vdev, n_cols=n, ld=ld)
    torch.cuda.synchronize()
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    got = idx.cpu().numpy()
    check_rows = range(rows) if rows <= 8 else sorted(set(np.random.default_rng(seed).integers(0, rows, 8)) | {0, rows - 1})
    for r in check_rows:
        vl = n if valid is None else int(valid[r])
        want = O.topk(sc[r], vl, k)
        assert np.array_equal(got[r], want), f"row {r}: first mismatch at {int(np.argmax(got[r] != want))}"


_CL_CASES = [c for c in CASES if c[2] <= (1 << 19)]


@pytest.mark.parametrize("kind,rows,n,k,mode", _CL_CASES, ids=[f"{c[0]}-{c[1]}x{c[2]}-k{c[3]}-{c[4]}" for c in _CL_CASES])
def test_topk_collect_select_path_equals_cluster_path(kind, rows, n, k, mode, test_hooks):
    """Rows of up to 2^19 positions take the one-cluster-per-row kernel; the
    collect + per-row select kernel (the path of longer rows, forced here by
    the test build) gives the same index arrays."""
    from sparse_attention_decode_scan_b200 import lsa
    seed = 900 + rows + n % 97 + k
    sc = synth.topk_scores(kind, rows, n, seed)
    valid = _valid(mode, rows, n, seed)
    ld = (n + 3) // 4 * 4
    dev = torch.full((rows, ld), float("nan"), dtype=torch.float32, device="cuda")
    dev[:, :n] = torch.from_numpy(sc).cuda()
    vdev = torch.from_numpy(valid).cuda() if valid is not None else None
    got = []
    for no_cluster in (False, True):
        test_hooks(no_cluster_topk=no_cluster)
        idx = torch.full((rows, k), -7, dtype=torch.int32, device="cuda")
        ws = lsa.workspace(lsa.topk_workspace_size(rows, n, k))
        lsa.topk(dev, k, idx, ws, valid_len=vdev, n_cols=n, ld=ld)
        torch.cuda.synchronize()
        assert lsa.read_device_status(ws) == lsa.LSA_OK
        got.append(idx.cpu().numpy())
    assert np.array_equal(got[0], got[1])


def test_topk_repeatable_and_workspace_reuse():
    from sparse_attention_decode_scan_b200 import lsa
    rows, n, k = 6, 50000, 2048
    sc = synth.topk_scores("ties", rows, n, 31)
    dev = torch.from_numpy(sc).cuda()
    ws = lsa.workspace(lsa.topk_workspace_size(rows, n, k))
    outs = []
    for _ in range(3):
        idx = torch.empty((rows, k), dtype=torch.int32, device="cuda")
        lsa.topk(dev, k, idx, ws)
        outs.append(idx.cpu().numpy())
    assert all(np.array_equal(outs[0], o) for o in outs[1:])
    for r in range(rows):
        assert np.array_equal(outs[0][r], O.topk(sc[r], n, k))
