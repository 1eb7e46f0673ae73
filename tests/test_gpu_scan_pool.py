"""The decode scan's pooled tile schedule.

With a pool (test build only: the library's default is the static split),
the decode step's scan CTAs take an even share of most tiles and claim the
rest from a counter in small chunks.  Which CTA scores a tile does not change
how the tile is scored, so every schedule must give bitwise the same step:
selection, output and lse.  The
schedules below cover no pool at all, the default, every tile from the pool
one at a time (the most segments, each CTA's first segment from the pool),
chunks that cross rows, and a pool that is empty from the start (every CTA's
first claim is past the end).
"""
import numpy as np
import pytest

from oracle import lsa_oracle as O
from sparse_attention_decode_scan_b200 import synth
from tests import cases
from tests.helpers import check_selection
from tests.test_gpu_step import _check_step, _step

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

# (static thousandths, tiles per claim); > 1000: no pool
NO_POOL = (1001, 0)
SCHEDULES = [(900, 4), (0, 1), (0, 4), (500, 3), (1000, 4), (950, 2)]


def _mid_case():
    """Paged bf16 decode with about 11 tiles per scan CTA: several pooled
    segments per CTA, chunks crossing from one sequence into the next."""
    spec = synth.scaled(synth.WORKLOADS[synth.DECODE_B32], batch=8, len_lo=15000, len_hi=30000, top_k=512)
    return synth.make_case(spec, 7301)


def _equal_steps(dc, scan_pool, schedules):
    scan_pool(*NO_POOL)
    o0, l0, i0 = _step(dc)
    for sched in schedules:
        scan_pool(*sched)
        o, l, i = _step(dc)
        assert torch.equal(i, i0), f"selection differs under schedule {sched}"
        assert torch.equal(o, o0), f"output differs under schedule {sched}"
        assert torch.equal(l, l0), f"lse differs under schedule {sched}"


@pytest.mark.parametrize("name", ["bf16_L5000", "paged_B5", "fp8_L6001", "len1"])
def test_pooled_step_bitwise_equals_static(name, scan_pool):
    from sparse_attention_decode_scan_b200.device import DeviceCase
    _equal_steps(DeviceCase(cases.small(name)), scan_pool, SCHEDULES)


def test_pooled_step_mid_size(scan_pool):
    """Bitwise equality on the mid-size case, and a pooled schedule's
    selection on two rows against the oracle."""
    from sparse_attention_decode_scan_b200.device import DeviceCase
    case = _mid_case()
    dc = DeviceCase(case)
    _equal_steps(dc, scan_pool, SCHEDULES)
    scan_pool(900, 4)
    _, _, idx = _step(dc)
    idx_h = idx.cpu().numpy()
    for r in (0, case.rows - 1):
        sc = O.row_scores(case, r)
        ref = O.topk(sc, O.row_visible(case, r), case.spec.top_k)
        check_selection(idx_h[r], ref, sc, what=f"mid case row {r}")


def test_pooled_step_vs_oracle_all_pooled(scan_pool):
    """Every tile from the pool, one per claim: the step against the oracle."""
    scan_pool(0, 1)
    case = cases.small("paged_B5")
    _check_step(case, list(range(case.rows)))


@pytest.mark.slow
@pytest.mark.parametrize("name", [synth.DECODE_B1, synth.DECODE_B32, synth.DECODE_B4_FP8])
def test_pooled_step_full_bitwise_equals_static(name, scan_pool):
    from sparse_attention_decode_scan_b200.device import DeviceCase
    _equal_steps(DeviceCase(cases.full(name)), scan_pool, [(900, 4), (0, 1)])
