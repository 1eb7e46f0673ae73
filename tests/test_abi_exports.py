"""The C-ABI library loads and exports every entry point include/lsa.h declares.

CPU only: besides symbol lookup, it calls only entry points that do no CUDA
work (version, status strings, workspace sizing, host-side argument checks that
return before anything is enqueued).
"""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lsa.h")
TEST_HEADER = os.path.join(ROOT, "include", "lsa_test.h")


@pytest.fixture(scope="module")
def lsa():
    from sparse_attention_decode_scan_b200 import build
    build.build()
    from sparse_attention_decode_scan_b200 import lsa as binding
    binding.lib()
    return binding


def declared_functions(header=HEADER):
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(lsa_[a-z_]+)\s*\(", text)))


def test_header_declares_the_step_entry_points():
    names = declared_functions()
    for n in ["lsa_indexer_scores", "lsa_topk", "lsa_sparse_attn_decode", "lsa_decode_step",
              "lsa_workspace_size", "lsa_read_device_status", "lsa_status_string", "lsa_version"]:
        assert n in names


def test_every_declared_symbol_is_exported(lsa):
    lib = lsa.lib()
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in lsa.h but not exported"


def test_test_library_exports_both_headers_and_the_product_no_switch(lsa):
    """liblsa_test.so exports lsa.h and lsa_test.h; liblsa.so exports nothing of lsa_test.h."""
    import ctypes as C
    test_only = declared_functions(TEST_HEADER)
    assert test_only == ["lsa_test_set_hooks", "lsa_test_set_scan_pool"]
    prod = C.CDLL(lsa.LIB_PATH)
    for n in test_only:
        assert not hasattr(prod, n), f"{n} must exist only in the test build"
    test_lib = C.CDLL(lsa.TEST_LIB_PATH)
    for n in declared_functions() + test_only:
        assert hasattr(test_lib, n), f"{n} not exported by liblsa_test.so"


def test_product_library_reads_no_environment():
    """The product path has no environment switch: no source of the library calls getenv."""
    import glob
    for f in glob.glob(os.path.join(ROOT, "sparse_attention_decode_scan_b200", "csrc", "*")):
        assert "getenv" not in open(f).read(), f"{os.path.basename(f)} reads the environment"


def test_version_and_status_strings(lsa):
    assert lsa.version() == 1
    assert lsa.status_string(lsa.LSA_OK) == "ok"
    assert "workspace" in lsa.status_string(lsa.LSA_ERR_WORKSPACE)
    assert lsa.status_string(99) == "unknown status"


def _dims(lsa, **kw):
    from sparse_attention_decode_scan_b200 import synth
    from sparse_attention_decode_scan_b200.device import make_dims
    d = make_dims(synth.WORKLOADS[synth.DECODE_B32])
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_workspace_sizes(lsa):
    d = _dims(lsa)
    step = lsa.workspace_size(d, 32, 131072, lsa.LSA_OP_DECODE_STEP)
    # at least: status + fp32 scores + selection
    assert step >= 256 + 32 * 131072 * 4 + 32 * 2048 * 4
    assert step % 256 == 0
    assert lsa.topk_workspace_size(4, 524288, 2048) > 0
    assert lsa.workspace_size(None, 4, 524288, lsa.LSA_OP_TOPK) == 0
    assert lsa.workspace_size(_dims(lsa, n_idx_heads=0), 1, 10, lsa.LSA_OP_DECODE_STEP) == 0
    assert lsa.workspace_size(d, -1, 10, lsa.LSA_OP_ATTN) == 0
    assert lsa.workspace_size(d, 1, 10, 99) == 0


def test_host_side_rejections_without_cuda(lsa):
    lib = lsa.lib()
    # invalid arguments return before any CUDA call
    assert lib.lsa_topk(None, 8, -1, None, 8, 4, None, None, 0, None) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_topk(None, 6, 1, None, 8, 4, None, None, 0, None) == lsa.LSA_ERR_INVALID_ARG  # ld < n
    d = _dims(lsa, idx_dim=12)  # not a multiple of 8
    c = lsa.Cache()
    assert lib.lsa_indexer_scores(ctypes.byref(d), ctypes.byref(c), 1, None, None, None, None, None, 8, None,
                                  0, None) == lsa.LSA_ERR_INVALID_ARG
    d = _dims(lsa)
    assert lib.lsa_decode_step(ctypes.byref(d), None, None, None, None, None, None, None, 0, None, 0,
                               None) == lsa.LSA_ERR_INVALID_ARG
    st = ctypes.c_int32(0)
    assert lib.lsa_read_device_status(None, ctypes.byref(st), None) == lsa.LSA_ERR_INVALID_ARG
    assert lib.lsa_get_device_status(None, None) == lsa.LSA_ERR_INVALID_ARG
