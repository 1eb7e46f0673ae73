"""Parity criteria shared by the GPU tests (the CPU oracle is the reference).

Tolerances:
  * indexer scores: |I_gpu - I_ref| <= tol * max(|I_ref(s)|, 1e-2 * max_s' |I_ref(s')|),
    tol = 1e-3 for bf16/fp32 keys, 2e-2 for FP8 keys; masked entries are -inf exactly;
  * top-k on fixed fp32 scores: identical index arrays;
  * end-to-end selection: equal sizes, and every position in the symmetric
    difference has an oracle score within 1e-3 relative of the oracle's k-th score;
  * attention: max |o_gpu - o_ref| <= 1e-2 with o_gpu cast to fp32, given the same
    selection (the GPU attention is run on the oracle's selection); lse within 1e-2.
"""
import numpy as np

SCORE_TOL = {"f32": 1e-3, "bf16": 1e-3, "fp8": 2e-2}
SEL_TOL = 1e-3
ATTN_TOL = 1e-2


def check_scores(gpu: np.ndarray, ref: np.ndarray, tol: float, what: str = "") -> float:
    """gpu fp32 row(s) vs oracle fp64 row(s) over the same positions; returns worst ratio."""
    gpu = np.asarray(gpu, np.float64)
    ref = np.asarray(ref, np.float64)
    masked = np.isneginf(ref)
    assert np.array_equal(np.isneginf(gpu), masked), f"{what}: -inf mask differs"
    assert np.isfinite(gpu[~masked]).all(), f"{what}: non-finite score"
    if (~masked).sum() == 0:
        return 0.0
    r = ref[~masked]
    g = gpu[~masked]
    floor = 1e-2 * np.abs(r).max()
    bound = tol * np.maximum(np.abs(r), floor)
    ratio = np.abs(g - r) / np.where(bound > 0, bound, 1.0)
    worst = float(ratio.max())
    assert worst <= 1.0, f"{what}: score error {worst:.3g}x tolerance at position {int(np.argmax(ratio))}"
    return worst


def check_selection(gpu_sel: np.ndarray, ref_sel: np.ndarray, ref_scores: np.ndarray, what: str = "") -> int:
    """Returns the size of the symmetric difference (all of it within the near-tie window)."""
    g = set(int(x) for x in gpu_sel if x >= 0)
    r = set(int(x) for x in ref_sel if x >= 0)
    assert len(g) == len(r), f"{what}: selection sizes {len(g)} vs {len(r)}"
    g_arr = np.asarray(gpu_sel)
    n = len(g)
    assert (g_arr[:n] >= 0).all() and (g_arr[n:] == -1).all(), f"{what}: padding not at the end"
    assert (np.diff(g_arr[:n]) > 0).all(), f"{what}: selection not strictly ascending"
    diff = g ^ r
    if diff:
        kth = ref_scores[sorted(r)].min()
        for s in diff:
            assert abs(ref_scores[s] - kth) <= SEL_TOL * abs(kth), \
                f"{what}: position {s} (score {ref_scores[s]}) differs outside the tie window of {kth}"
    return len(diff)


def check_attention(o_gpu, o_ref, lse_gpu=None, lse_ref=None, what: str = "") -> float:
    o_gpu = np.asarray(o_gpu, np.float64)
    err = float(np.abs(o_gpu - o_ref).max()) if o_ref.size else 0.0
    assert err <= ATTN_TOL, f"{what}: attention max-abs error {err}"
    if lse_gpu is not None and lse_ref is not None:
        lg, lr = np.asarray(lse_gpu, np.float64), np.asarray(lse_ref, np.float64)
        inf = np.isneginf(lr)
        assert np.array_equal(np.isneginf(lg), inf), f"{what}: lse -inf mask differs"
        if (~inf).any():
            e2 = float(np.abs(lg[~inf] - lr[~inf]).max())
            assert e2 <= ATTN_TOL, f"{what}: lse error {e2}"
    return err
