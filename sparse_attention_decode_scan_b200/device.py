"""Device-resident copies of a synthetic case, with the C-ABI structs that
describe them (plumbing only: copies and pointer bookkeeping)."""
from __future__ import annotations

import numpy as np

from . import lsa


def to_device(arr: np.ndarray, dtype: str, device="cuda", pin: bool = False):
    """numpy storage (fp32 / bf16 bits / e4m3 bits / int32) -> torch tensor on `device`."""
    import torch
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    elif dtype == "fp8":
        t = torch.from_numpy(np.ascontiguousarray(arr)).view(torch.float8_e4m3fn)
    else:
        t = torch.from_numpy(np.ascontiguousarray(arr))
    if pin:
        return t.pin_memory()
    return t.to(device)


class DeviceCase:
    """A synth.Case on the GPU plus its lsa Dims / Cache structs."""

    def __init__(self, case, device="cuda", top_k=None, share: "DeviceCase" = None):
        """`share`: another layer of the same batch whose lengths, block table
        and row map (the same arrays) this layer's cache struct points at."""
        import torch
        s = case.spec
        self.case = case
        self.spec = s
        self.device = device
        if share is not None:
            assert np.array_equal(case.seq_lens, share.case.seq_lens)
            self.seq_lens, self.block_table = share.seq_lens, share.block_table
        else:
            self.seq_lens = torch.from_numpy(case.seq_lens).to(device)
            self.block_table = torch.from_numpy(case.block_table).to(device) if case.block_table is not None else None
        self.idx_keys = to_device(case.idx_keys, s.idx_key_dtype, device)
        self.idx_scales = torch.from_numpy(case.idx_scales).to(device) if case.idx_scales is not None else None
        self.kv = to_device(case.kv, s.act_dtype, device) if case.kv is not None else None
        self.row_seq = torch.from_numpy(case.row_seq).to(device)
        self.row_pos = torch.from_numpy(case.row_pos).to(device) if case.row_pos is not None else None
        self.q_idx = to_device(case.q_idx, s.act_dtype, device)
        self.w = torch.from_numpy(case.w).to(device)
        self.q = to_device(case.q, s.act_dtype, device) if case.q is not None else None
        self.max_len = int(s.stride if s.block_size == 0 else case.max_blocks * s.block_size)
        self.dims = make_dims(s, top_k)
        self.cache = self.make_cache()

    def make_cache(self) -> lsa.Cache:
        s = self.spec
        c = lsa.Cache()
        c.idx_keys = self.idx_keys.data_ptr()
        c.idx_key_scales = self.idx_scales.data_ptr() if self.idx_scales is not None else None
        c.kv = self.kv.data_ptr() if self.kv is not None else None
        c.block_table = self.block_table.data_ptr() if self.block_table is not None else None
        c.max_blocks_per_seq = self.case.max_blocks
        c.n_blocks = int(self.idx_keys.shape[0]) if s.block_size else 0
        c.max_len = self.max_len
        c.seq_lens = self.seq_lens.data_ptr()
        c.batch = int(self.seq_lens.shape[0])
        return c

    @property
    def rows(self) -> int:
        return int(self.row_seq.shape[0])


def make_dims(s, top_k=None) -> lsa.Dims:
    d = lsa.Dims()
    d.n_idx_heads = s.n_idx_heads
    d.idx_dim = s.idx_dim
    d.n_heads = s.n_heads
    d.qk_dim = s.qk_dim
    d.v_dim = s.v_dim
    d.top_k = s.top_k if top_k is None else top_k
    d.block_size = s.block_size
    d.softmax_scale = s.softmax_scale
    d.act_dtype = lsa.DTYPE_CODE[s.act_dtype]
    d.idx_key_dtype = lsa.DTYPE_CODE[s.idx_key_dtype]
    return d


def device_layers(cases, device="cuda"):
    """DeviceCases of the layers of one batch, sharing layer 0's lengths and block table."""
    first = DeviceCase(cases[0], device=device)
    return [first] + [DeviceCase(c, device=device, share=first) for c in cases[1:]]
