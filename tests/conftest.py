import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200) and the built liblsa.so")
    config.addinivalue_line("markers", "slow: full-size workload")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_gpu = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_gpu = False
    if has_gpu:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for it in items:
        if "gpu" in it.keywords:
            it.add_marker(skip)


@pytest.fixture
def test_hooks():
    """Routes the binding to liblsa_test.so (the product library has no switches) and yields its
    hook setter; restores the defaults and the product library afterwards."""
    from sparse_attention_decode_scan_b200 import lsa
    lsa.use_test_library(True)
    try:
        yield lsa.set_test_hooks
    finally:
        lsa.set_test_hooks()
        lsa.use_test_library(False)


@pytest.fixture
def scan_pool():
    """Routes the binding to liblsa_test.so and yields its scan-schedule setter
    (lsa_test_set_scan_pool); restores the default schedule and the product
    library afterwards."""
    from sparse_attention_decode_scan_b200 import lsa
    lsa.use_test_library(True)
    try:
        yield lsa.set_test_scan_pool
    finally:
        lsa.set_test_scan_pool()
        lsa.use_test_library(False)
