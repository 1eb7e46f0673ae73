"""Thin ctypes binding of liblsa.so (C ABI in include/lsa.h).

Argument marshalling only: torch tensors are passed as raw device pointers with
the current CUDA stream; every step of the computation runs in the library's
CUDA kernels.  There is no fallback: if liblsa.so is missing or fails to load,
importing the binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsa.so")
# Test build (include/lsa_test.h): the same kernels plus lsa_test_set_hooks.
TEST_LIB_PATH = os.path.join(_HERE, "liblsa_test.so")

LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_UNSUPPORTED, LSA_ERR_WORKSPACE, LSA_ERR_CUDA, LSA_ERR_TIMEOUT, \
    LSA_ERR_BOUNDS = range(7)
LSA_F32, LSA_BF16, LSA_FP8_E4M3 = 0, 1, 2
LSA_OP_SCORES, LSA_OP_TOPK, LSA_OP_ATTN, LSA_OP_DECODE_STEP, LSA_OP_DECODE_STEP_FUSED, LSA_OP_DECODE_LAYERS = \
    0, 1, 2, 3, 4, 5
LSA_STEP_UNFUSED, LSA_STEP_FUSED = 0, 1
LSA_ROUTE_OWN, LSA_ROUTE_PREV = 0, 1

DTYPE_CODE = {"f32": LSA_F32, "bf16": LSA_BF16, "fp8": LSA_FP8_E4M3}


class LsaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (lsa_status {code})")


class Dims(ctypes.Structure):
    _fields_ = [("n_idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("n_heads", ctypes.c_int32), ("qk_dim", ctypes.c_int32), ("v_dim", ctypes.c_int32),
                ("top_k", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("act_dtype", ctypes.c_int32),
                ("idx_key_dtype", ctypes.c_int32)]


class Cache(ctypes.Structure):
    _fields_ = [("idx_keys", ctypes.c_void_p), ("idx_key_scales", ctypes.c_void_p),
                ("kv", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("max_blocks_per_seq", ctypes.c_int32), ("n_blocks", ctypes.c_int64),
                ("max_len", ctypes.c_int64), ("seq_lens", ctypes.c_void_p), ("batch", ctypes.c_int32)]


_libs = {}
_use_test = False


def use_test_library(on: bool = True) -> None:
    """Routes every later call of this binding to liblsa_test.so (on) or back to liblsa.so.
    Only tests do this, to reach lsa_test_set_hooks."""
    global _use_test
    _use_test = bool(on)


def set_test_hooks(force_simt: bool = False, split_select_min_cols: int = -1, scan_wait_extra: int = 0,
                   no_cluster_topk: bool = False) -> None:
    """lsa_test_set_hooks of liblsa_test.so (include/lsa_test.h); needs use_test_library()."""
    if not _use_test:
        raise RuntimeError("test hooks exist only in liblsa_test.so: call use_test_library() first")
    _check(lib().lsa_test_set_hooks(1 if force_simt else 0, int(split_select_min_cols), int(scan_wait_extra),
                                    1 if no_cluster_topk else 0), "lsa_test_set_hooks")


def set_test_scan_pool(static_pm: int = -1, chunk: int = 0) -> None:
    """lsa_test_set_scan_pool of liblsa_test.so (include/lsa_test.h); needs use_test_library()."""
    if not _use_test:
        raise RuntimeError("test hooks exist only in liblsa_test.so: call use_test_library() first")
    _check(lib().lsa_test_set_scan_pool(int(static_pm), int(chunk)), "lsa_test_set_scan_pool")


def lib() -> ctypes.CDLL:
    """Loads liblsa.so (or, after use_test_library(), liblsa_test.so) once; raises if it is absent
    (no fallback path exists)."""
    path = TEST_LIB_PATH if _use_test else LIB_PATH
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} not built at {path}; run "
                          "`python -m sparse_attention_decode_scan_b200.build`")
    L = ctypes.CDLL(path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    D, C = ctypes.POINTER(Dims), ctypes.POINTER(Cache)
    L.lsa_workspace_size.argtypes = [D, i32, i64, i32]
    L.lsa_workspace_size.restype = sz
    L.lsa_indexer_scores.argtypes = [D, C, i32, vp, vp, vp, vp, vp, i64, vp, sz, vp]
    L.lsa_topk.argtypes = [vp, i64, i32, vp, i64, i32, vp, vp, sz, vp]
    L.lsa_topk_noalloc.argtypes = [vp, i64, i32, vp, i64, i32, vp, vp]
    L.lsa_sparse_attn_decode.argtypes = [D, C, i32, vp, vp, vp, vp, vp, vp, sz, vp]
    L.lsa_decode_step.argtypes = [D, C, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp]
    L.lsa_decode_step_profiled.argtypes = [D, C, vp, vp, vp, vp, vp, vp, i32, vp, sz, vp, ctypes.POINTER(vp)]
    PV = ctypes.POINTER(vp)
    L.lsa_decode_layers.argtypes = [D, i32, C, PV, PV, PV, PV, PV, i32, i32, vp, vp, sz, vp]
    L.lsa_read_device_status.argtypes = [vp, ctypes.POINTER(i32), vp]
    L.lsa_get_device_status.argtypes = [vp, vp]
    L.lsa_status_string.argtypes = [ctypes.c_int]
    L.lsa_status_string.restype = ctypes.c_char_p
    L.lsa_version.restype = i32
    L.lsa_launch_count.argtypes = [D, i32, i64, i32, i32]
    L.lsa_launch_count.restype = i32
    L.lsa_candidate_scores.argtypes = [D, C, i32, vp, vp, vp, vp, vp, i32, vp, i64, vp, sz, vp]
    L.lsa_two_stage_workspace_size.argtypes = [D, i32, i64, i32]
    L.lsa_two_stage_workspace_size.restype = sz
    L.lsa_two_stage_select.argtypes = [D, C, vp, vp, i32, vp, vp, vp, vp, i32, vp, vp, sz, vp]
    L.lsa_block_select_workspace_size.argtypes = [i32, i64, i32, i32]
    L.lsa_block_select_workspace_size.restype = sz
    L.lsa_block_select.argtypes = [vp, i64, i32, vp, i64, i32, i32, vp, vp, sz, vp]
    L.lsa_stage_blocks.argtypes = [D, C, i32, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp]
    L.lsa_prefill_layers_workspace_size.argtypes = [D, i32, i64, i32]
    L.lsa_prefill_layers_workspace_size.restype = sz
    L.lsa_prefill_layers.argtypes = [D, i32, C, i64, PV, i32, vp, PV, PV, PV, PV, PV, PV, i32, PV, vp, sz, vp, vp, PV]
    names = ["lsa_prefill_layers", "lsa_indexer_scores", "lsa_topk", "lsa_topk_noalloc", "lsa_sparse_attn_decode",
             "lsa_decode_step",
             "lsa_decode_step_profiled", "lsa_decode_layers", "lsa_read_device_status", "lsa_get_device_status",
             "lsa_candidate_scores",
             "lsa_two_stage_select", "lsa_block_select", "lsa_stage_blocks"]
    if path == TEST_LIB_PATH:
        L.lsa_test_set_hooks.argtypes = [i32, i64, ctypes.c_uint32, i32]
        L.lsa_test_set_scan_pool.argtypes = [i32, i32]
        names += ["lsa_test_set_hooks", "lsa_test_set_scan_pool"]
    for f in names:
        getattr(L, f).restype = ctypes.c_int
    _libs[path] = L
    return L


def status_string(code: int) -> str:
    return lib().lsa_status_string(int(code)).decode()


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return int(t.data_ptr())


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _check(code: int, where: str, raise_on_error: bool = True) -> int:
    if code != LSA_OK and raise_on_error:
        raise LsaError(code, where)
    return code


def workspace_size(dims: Optional[Dims], rows: int, max_len: int, op: int) -> int:
    return int(lib().lsa_workspace_size(ctypes.byref(dims) if dims is not None else None, rows, max_len, op))


def topk_workspace_size(rows: int, n_cols: int, k: int) -> int:
    """Workspace bytes of lsa_topk for these sizes (only k of the dims is read)."""
    d = Dims()
    d.top_k = int(k)
    return workspace_size(d, rows, n_cols, LSA_OP_TOPK)


def workspace(nbytes: int, device="cuda"):
    """A zero-filled, 256-byte aligned workspace tensor (torch's allocator aligns to 512 B)."""
    import torch
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def indexer_scores(dims: Dims, cache: Cache, q_idx, w, scores, ld: int, ws, row_seq=None, row_pos=None,
                   rows: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    rows = int(q_idx.shape[0]) if rows is None else rows
    return _check(lib().lsa_indexer_scores(ctypes.byref(dims), ctypes.byref(cache), rows, _ptr(row_seq),
                                           _ptr(row_pos), _ptr(q_idx), _ptr(w), _ptr(scores), int(ld),
                                           _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)),
                  "lsa_indexer_scores", raise_on_error)


def topk(scores, k: int, idx, ws, valid_len=None, n_cols: Optional[int] = None, ld: Optional[int] = None,
         rows: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    rows = int(scores.shape[0]) if rows is None else rows
    ld = int(scores.stride(0)) if ld is None else ld
    n_cols = int(scores.shape[1]) if n_cols is None else n_cols
    return _check(lib().lsa_topk(_ptr(scores), ld, rows, _ptr(valid_len), n_cols, int(k), _ptr(idx), _ptr(ws),
                                 ws.numel() if ws is not None else 0, _stream(stream)),
                  "lsa_topk", raise_on_error)


def topk_noalloc(scores, k: int, idx, valid_len=None, n_cols: Optional[int] = None, ld: Optional[int] = None,
                 rows: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    """lsa_topk_noalloc: the top-k with the library's static scratch instead of a workspace."""
    rows = int(scores.shape[0]) if rows is None else rows
    ld = int(scores.stride(0)) if ld is None else ld
    n_cols = int(scores.shape[1]) if n_cols is None else n_cols
    return _check(lib().lsa_topk_noalloc(_ptr(scores), ld, rows, _ptr(valid_len), n_cols, int(k), _ptr(idx),
                                         _stream(stream)), "lsa_topk_noalloc", raise_on_error)


def sparse_attn_decode(dims: Dims, cache: Cache, q, idx, out, lse, ws, row_seq=None, rows: Optional[int] = None,
                       stream=None, raise_on_error=True) -> int:
    rows = int(q.shape[0]) if rows is None else rows
    return _check(lib().lsa_sparse_attn_decode(ctypes.byref(dims), ctypes.byref(cache), rows, _ptr(row_seq),
                                               _ptr(q), _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws),
                                               ws.numel() if ws is not None else 0, _stream(stream)),
                  "lsa_sparse_attn_decode", raise_on_error)


def decode_step(dims: Dims, cache: Cache, q_idx, w, q, out, lse, ws, idx_out=None, flags: int = LSA_STEP_UNFUSED,
                stream=None, raise_on_error=True) -> int:
    return _check(lib().lsa_decode_step(ctypes.byref(dims), ctypes.byref(cache), _ptr(q_idx), _ptr(w), _ptr(q),
                                        _ptr(out), _ptr(lse), _ptr(idx_out), int(flags), _ptr(ws),
                                        ws.numel() if ws is not None else 0, _stream(stream)),
                  "lsa_decode_step", raise_on_error)


def decode_step_profiled(dims: Dims, cache: Cache, q_idx, w, q, out, lse, ws, events, idx_out=None,
                         flags: int = LSA_STEP_UNFUSED, stream=None, raise_on_error=True) -> int:
    """lsa_decode_step recording 4 CUDA events (torch.cuda.Event, already created) at phase boundaries."""
    ev = (ctypes.c_void_p * 4)(*[int(e.cuda_event) if e is not None else None for e in events])
    return _check(lib().lsa_decode_step_profiled(ctypes.byref(dims), ctypes.byref(cache), _ptr(q_idx), _ptr(w),
                                                 _ptr(q), _ptr(out), _ptr(lse), _ptr(idx_out), int(flags),
                                                 _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream),
                                                 ev), "lsa_decode_step_profiled", raise_on_error)


def decode_layers(dims: Dims, caches, q_idx, w, q, out, lse, ws, retention: int = 1, route: int = LSA_ROUTE_OWN,
                  idx_out=None, stream=None, raise_on_error=True) -> int:
    """lsa_decode_layers: per-layer lists of Cache structs and tensors (q_idx / w entries may be None for
    layers without an indexer, lse may be None)."""
    n = len(caches)
    arr = (Cache * n)(*caches)

    def ptrs(ts):
        return (ctypes.c_void_p * n)(*[_ptr(t) for t in ts]) if ts is not None else None

    return _check(lib().lsa_decode_layers(ctypes.byref(dims), n, arr, ptrs(q_idx), ptrs(w), ptrs(q), ptrs(out),
                                          ptrs(lse), int(retention), int(route), _ptr(idx_out), _ptr(ws),
                                          ws.numel() if ws is not None else 0, _stream(stream)),
                  "lsa_decode_layers", raise_on_error)


def candidate_scores(dims: Dims, cache: Cache, q_idx, w, cand, scores, ld: int, ws, row_seq=None, row_pos=None,
                     rows: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    """lsa_candidate_scores: exact scores of the positions cand [rows, n_cand] into scores [rows, ld]."""
    rows = int(q_idx.shape[0]) if rows is None else rows
    n_cand = int(cand.shape[1])
    return _check(lib().lsa_candidate_scores(ctypes.byref(dims), ctypes.byref(cache), rows, _ptr(row_seq),
                                             _ptr(row_pos), _ptr(q_idx), _ptr(w), _ptr(cand), n_cand, _ptr(scores),
                                             int(ld), _ptr(ws), ws.numel() if ws is not None else 0,
                                             _stream(stream)), "lsa_candidate_scores", raise_on_error)


def two_stage_workspace_size(dims: Dims, rows: int, max_len: int, n_cand: int) -> int:
    return int(lib().lsa_two_stage_workspace_size(ctypes.byref(dims), rows, max_len, n_cand))


def two_stage_select(dims: Dims, cache: Cache, compact_keys, compact_scales, q_idx, w, n_cand: int, idx, ws,
                     row_seq=None, row_pos=None, rows: Optional[int] = None, stream=None,
                     raise_on_error=True) -> int:
    """lsa_two_stage_select: the k = dims.top_k selection of each row by the two-stage search."""
    rows = int(q_idx.shape[0]) if rows is None else rows
    return _check(lib().lsa_two_stage_select(ctypes.byref(dims), ctypes.byref(cache), _ptr(compact_keys),
                                             _ptr(compact_scales), rows, _ptr(row_seq), _ptr(row_pos), _ptr(q_idx),
                                             _ptr(w), int(n_cand), _ptr(idx), _ptr(ws),
                                             ws.numel() if ws is not None else 0, _stream(stream)),
                  "lsa_two_stage_select", raise_on_error)


def block_select_workspace_size(rows: int, n_cols: int, block_size: int, n_sel: int) -> int:
    return int(lib().lsa_block_select_workspace_size(rows, n_cols, block_size, n_sel))


def block_select(scores, block_size: int, n_sel: int, kept, ws, valid_len=None, n_cols: Optional[int] = None,
                 ld: Optional[int] = None, rows: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    """lsa_block_select: kept [rows, n_sel] block ids from scores [rows, ld]."""
    rows = int(scores.shape[0]) if rows is None else rows
    ld = int(scores.stride(0)) if ld is None else ld
    n_cols = int(scores.shape[1]) if n_cols is None else n_cols
    return _check(lib().lsa_block_select(_ptr(scores), ld, rows, _ptr(valid_len), n_cols, int(block_size),
                                         int(n_sel), _ptr(kept), _ptr(ws), ws.numel() if ws is not None else 0,
                                         _stream(stream)), "lsa_block_select", raise_on_error)


def stage_blocks(dims: Dims, cache: Cache, kept, block_size: int, staged_kv, staged_table, staged_idx, ws,
                 row_seq=None, row_pos=None, rows: Optional[int] = None, stream=None, raise_on_error=True) -> int:
    """lsa_stage_blocks: the kept blocks' KV rows into the staging pool (cache.kv may be pinned host memory)."""
    rows = int(kept.shape[0]) if rows is None else rows
    return _check(lib().lsa_stage_blocks(ctypes.byref(dims), ctypes.byref(cache), rows, _ptr(row_seq), _ptr(row_pos),
                                         _ptr(kept),
                                         int(kept.shape[1]), int(block_size), _ptr(staged_kv), _ptr(staged_table),
                                         _ptr(staged_idx), _ptr(ws), ws.numel() if ws is not None else 0,
                                         _stream(stream)), "lsa_stage_blocks", raise_on_error)


def staged_cache(staged_kv, staged_table, staged_lens, n_sel: int, block_size: int) -> Cache:
    """The lsa_cache over a staging pool that lsa_sparse_attn_decode reads after lsa_stage_blocks."""
    c = Cache()
    c.idx_keys = None
    c.idx_key_scales = None
    c.kv = staged_kv.data_ptr()
    c.block_table = staged_table.data_ptr()
    c.max_blocks_per_seq = int(n_sel)
    c.n_blocks = int(staged_table.numel())
    c.max_len = int(n_sel * block_size)
    c.seq_lens = staged_lens.data_ptr()
    c.batch = int(staged_table.shape[0])
    return c


def prefill_layers_workspace_size(dims: Dims, rows: int, max_len: int, row_block: int) -> int:
    return int(lib().lsa_prefill_layers_workspace_size(ctypes.byref(dims), rows, max_len, row_block))


def prefill_layers(dims: Dims, caches, hist_len: int, chunk_kv, row_pos, q_idx, w, q, out, lse, kv_buf, ws,
                   row_block: int, events, idx_out=None, stream=None, copy_stream=None, raise_on_error=True) -> int:
    """lsa_prefill_layers: per-layer lists of Cache structs (kv = the history, host or device) and tensors;
    kv_buf: two device buffers; events: four torch.cuda.Event (created here if needed)."""
    import torch
    n = len(caches)
    arr = (Cache * n)(*caches)

    def ptrs(ts):
        return (ctypes.c_void_p * n)(*[_ptr(t) for t in ts]) if ts is not None else None

    for e in events:  # torch creates the CUDA event at its first record
        if e.cuda_event == 0:
            e.record()
    ev = (ctypes.c_void_p * 4)(*[int(e.cuda_event) for e in events])
    bufs = (ctypes.c_void_p * 2)(*[_ptr(t) for t in kv_buf])
    cs = copy_stream if copy_stream is not None else torch.cuda.Stream()
    rows = int(row_pos.shape[0])
    return _check(lib().lsa_prefill_layers(ctypes.byref(dims), n, arr, int(hist_len), ptrs(chunk_kv), rows,
                                           _ptr(row_pos), ptrs(q_idx), ptrs(w), ptrs(q), ptrs(out), ptrs(lse),
                                           ptrs(idx_out), int(row_block), bufs, _ptr(ws),
                                           ws.numel() if ws is not None else 0, _stream(stream), _stream(cs), ev),
                  "lsa_prefill_layers", raise_on_error)


def read_device_status(ws, stream=None) -> int:
    st = ctypes.c_int32(0)
    _check(lib().lsa_read_device_status(_ptr(ws), ctypes.byref(st), _stream(stream)), "lsa_read_device_status")
    return int(st.value)


def get_device_status(ws, stream=None) -> int:
    """lsa_get_device_status: the workspace status word (cleared), or the read's own error code."""
    return int(lib().lsa_get_device_status(_ptr(ws), _stream(stream)))


def launch_count(dims: Optional[Dims], rows: int, max_len: int, op: int, causal: bool = False) -> int:
    return int(lib().lsa_launch_count(ctypes.byref(dims) if dims is not None else None, rows, max_len, op,
                                      1 if causal else 0))


def version() -> int:
    return int(lib().lsa_version())
