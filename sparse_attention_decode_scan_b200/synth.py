"""Seeded synthetic inputs for the DSA decode step and its causal prefill variant.

This module only draws random numbers and stores them in the element formats
the kernels read (fp32, bf16 bits, e4m3fn bits).  It computes nothing of the
method: no score, no selection, no softmax.  Both the CUDA path and the CPU
oracle receive the arrays built here, so the two sides see identical bytes.

Workloads follow the five shapes of the decode-step benchmark family:
a tiny fp32 step, one production-width bf16 sequence, a paged batch of 32
long sequences, FP8 indexer keys at 512K tokens, and a causal prefill chunk.

Recipe (every draw is independent and keyed by (seed, array name)):
  * normal entries ~ N(0, 1) in fp32, rounded to bf16 with round-to-nearest-even
    where the workload stores bf16;
  * indexer weights w ~ N(0, 1) * w_std, kept in fp32;
  * sequence lengths ~ U{len_lo .. len_hi};
  * paged caches: one physical block per logical block, physical ids are a
    random permutation of all blocks; unused block-table entries are -1;
  * FP8 keys: x ~ N(0, 1), a Bernoulli(heavy_frac) subset of tokens gets
    +heavy_offset on dimension 0, then x is clamped to the finite e4m3 range and
    rounded to e4m3fn (nearest-even); per-token scales ~ U[scale_lo, scale_hi];
  * cache rows past a sequence's length hold random data too (it must be
    ignored by every consumer).
"""
from __future__ import annotations

import math
import os
import zlib
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field, replace
from typing import Dict, List, Optional

import numpy as np

_CHUNK = 1 << 22  # elements per independent random stream


def _seedseq(seed: int, name: str) -> np.random.SeedSequence:
    return np.random.SeedSequence([int(seed), zlib.crc32(name.encode())])


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def normal(shape, seed: int, name: str, std: float = 1.0) -> np.ndarray:
    """fp32 N(0, std^2) array; chunked independent PCG64 streams, filled in threads."""
    n = int(np.prod(shape, dtype=np.int64))
    out = np.empty(n, np.float32)
    nch = max(1, (n + _CHUNK - 1) // _CHUNK)
    subs = _seedseq(seed, name).spawn(nch)

    def fill(i):
        g = np.random.Generator(np.random.PCG64(subs[i]))
        g.standard_normal(out=out[i * _CHUNK:(i + 1) * _CHUNK], dtype=np.float32)

    if nch == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nch)))
    if std != 1.0:
        out *= np.float32(std)
    return out.reshape(shape)


def rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(_seedseq(seed, name)))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round-to-nearest-even (torch's cast)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


E4M3_MAX = 448.0


def to_e4m3_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> e4m3fn bit patterns (uint8): clamp to +-448 (saturate to finite),
    then round-to-nearest-even (torch's float8_e4m3fn cast)."""
    import torch
    t = torch.from_numpy(np.clip(np.ascontiguousarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def encode(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    if dtype == "bf16":
        return to_bf16_bits(x)
    if dtype == "fp8":
        return to_e4m3_bits(x)
    raise ValueError(dtype)


@dataclass(frozen=True)
class Spec:
    """Shape and distribution of one workload.

    Decode: ``rows == batch`` (one query row per sequence, ``causal`` False).
    Prefill: one sequence whose last ``chunk`` cache tokens are the chunk's own
    keys; query row i sits at position ``len_lo - chunk + i`` and sees every
    position up to and including its own (``causal`` True).
    """
    name: str
    batch: int
    len_lo: int
    len_hi: int
    n_idx_heads: int
    idx_dim: int
    n_heads: int
    qk_dim: int
    v_dim: int
    top_k: int
    block_size: int = 0            # 0 = contiguous caches
    act_dtype: str = "bf16"        # q_idx, q, kv
    idx_key_dtype: str = "bf16"    # 'f32' | 'bf16' | 'fp8'
    w_std: float = 0.125
    softmax_scale: float = 1.0 / 24.0
    heavy_frac: float = 0.0
    heavy_offset: float = 0.0
    scale_lo: float = 0.5
    scale_hi: float = 2.0
    chunk: int = 0                 # prefill chunk rows (0 = decode)
    max_len: int = 0               # contiguous row stride; 0 -> len_hi
    with_kv: bool = True
    seed: int = 0                  # seed of the workload's data

    @property
    def streams_past_l2(self) -> bool:
        """The indexer keys of one step (bytes read by the scan) exceed twice
        the 126 MB L2, so consecutive steps need no L2 flush between them."""
        per_tok = {"f32": 4, "bf16": 2, "fp8": 1}[self.idx_key_dtype] * self.idx_dim + (
            4 if self.idx_key_dtype == "fp8" else 0)
        mean_len = (self.len_lo + self.len_hi) / 2
        return not self.causal and self.batch * mean_len * per_tok >= 2 * 126e6

    @property
    def causal(self) -> bool:
        return self.chunk > 0

    @property
    def stride(self) -> int:
        return self.max_len or self.len_hi


# The benchmark workloads, by name.  Each carries the seed its data is drawn
# with (every rank adds its own offset).
TINY = "tiny_fp32_L4096"
DECODE_B1 = "decode_B1_L32K_bf16"
DECODE_B32 = "decode_B32_L64K-128K_paged64_bf16"
DECODE_B4_FP8 = "decode_B4_L512K_fp8keys"
PREFILL = "prefill_8192x139264_causal_bf16"

WORKLOADS: Dict[str, Spec] = {s.name: s for s in [
    Spec(TINY, batch=1, len_lo=4096, len_hi=4096, n_idx_heads=4, idx_dim=64,
         n_heads=8, qk_dim=64, v_dim=64, top_k=256, act_dtype="f32", idx_key_dtype="f32",
         w_std=0.5, softmax_scale=1.0 / 8.0, seed=1001),
    Spec(DECODE_B1, batch=1, len_lo=32768, len_hi=32768, n_idx_heads=64,
         idx_dim=128, n_heads=128, qk_dim=576, v_dim=512, top_k=2048, seed=1002),
    Spec(DECODE_B32, batch=32, len_lo=65536, len_hi=131072,
         n_idx_heads=64, idx_dim=128, n_heads=128, qk_dim=576, v_dim=512, top_k=2048,
         block_size=64, seed=1003),
    Spec(DECODE_B4_FP8, batch=4, len_lo=524288, len_hi=524288, n_idx_heads=64,
         idx_dim=128, n_heads=128, qk_dim=576, v_dim=512, top_k=2048, idx_key_dtype="fp8",
         heavy_frac=0.1, heavy_offset=3.0, seed=1004),
    Spec(PREFILL, batch=1, len_lo=139264, len_hi=139264,
         n_idx_heads=64, idx_dim=128, n_heads=128, qk_dim=576, v_dim=512, top_k=2048,
         chunk=8192, seed=1005),
]}


def workload(name: str) -> Spec:
    """The workload called `name`, or the only one whose name starts with it."""
    if name in WORKLOADS:
        return WORKLOADS[name]
    hits = [k for k in WORKLOADS if k.startswith(name)]
    if len(hits) != 1:
        raise KeyError(f"workload {name!r}: {'ambiguous' if hits else 'unknown'} (one of {sorted(WORKLOADS)})")
    return WORKLOADS[hits[0]]


def seed_of(spec: Spec) -> int:
    return spec.seed


@dataclass
class Case:
    """Host arrays of one workload (numpy; bf16 as uint16 bits, fp8 as uint8 bits)."""
    spec: Spec
    seed: int
    seq_lens: np.ndarray                 # [B] int32
    block_table: Optional[np.ndarray]    # [B, max_blocks] int32 (-1 unused) or None
    idx_keys: np.ndarray                 # paged [n_blocks, bs, d_I] or [B, stride, d_I]
    idx_scales: Optional[np.ndarray]     # fp32 [n_blocks, bs] or [B, stride] (fp8 only)
    kv: Optional[np.ndarray]             # paged [n_blocks, bs, D] or [B, stride, D]
    row_seq: np.ndarray                  # [R] int32
    row_pos: Optional[np.ndarray]        # [R] int32 (causal) or None
    q_idx: np.ndarray                    # [R, H_I, d_I]
    w: np.ndarray                        # [R, H_I] fp32
    q: Optional[np.ndarray]              # [R, H, D]
    extra: dict = field(default_factory=dict)

    @property
    def rows(self) -> int:
        return int(self.row_seq.shape[0])

    @property
    def max_blocks(self) -> int:
        return 0 if self.block_table is None else int(self.block_table.shape[1])


def make_case(spec: Spec, seed: int, layer: int = 0) -> Case:
    """Host arrays of one workload.  `layer` > 0 draws another DSA layer of the
    same batch: the same sequence lengths and block table, its own cache
    contents and queries (layer 0 is the plain single-layer workload)."""
    s = spec
    tag = (lambda name: name) if layer == 0 else (lambda name: f"{name}@layer{layer}")
    r = rng(seed, "lengths")
    if s.causal:
        assert s.batch == 1 and s.len_lo == s.len_hi
    seq_lens = r.integers(s.len_lo, s.len_hi + 1, size=s.batch, dtype=np.int64).astype(np.int32)
    d_key = s.idx_dim
    key_dt = s.idx_key_dtype
    if s.block_size > 0:
        bs = s.block_size
        nb_seq = (seq_lens.astype(np.int64) + bs - 1) // bs
        n_blocks = int(nb_seq.sum())
        max_blocks = int((s.len_hi + bs - 1) // bs)
        perm = rng(seed, "block_perm").permutation(n_blocks).astype(np.int32)
        bt = np.full((s.batch, max_blocks), -1, np.int32)
        o = 0
        for b in range(s.batch):
            bt[b, :nb_seq[b]] = perm[o:o + nb_seq[b]]
            o += int(nb_seq[b])
        lead = (n_blocks, bs)
    else:
        bt = None
        lead = (s.batch, s.stride)
    ntok = int(np.prod(lead))
    keys_f = normal(lead + (d_key,), seed, tag("idx_keys"))
    scales = None
    if key_dt == "fp8":
        if s.heavy_frac > 0:
            heavy = rng(seed, tag("heavy")).random(ntok, dtype=np.float64) < s.heavy_frac
            keys_f.reshape(ntok, d_key)[heavy, 0] += np.float32(s.heavy_offset)
        scales = rng(seed, tag("idx_scales")).uniform(s.scale_lo, s.scale_hi, size=ntok).astype(np.float32)
        scales = scales.reshape(lead)
    idx_keys = encode(keys_f, key_dt)
    del keys_f
    kv = None
    if s.with_kv:
        kv = encode(normal(lead + (s.qk_dim,), seed, tag("kv")), s.act_dtype)
    if s.causal:
        R = s.chunk
        row_seq = np.zeros(R, np.int32)
        row_pos = (int(seq_lens[0]) - s.chunk + np.arange(R)).astype(np.int32)
    else:
        R = s.batch
        row_seq = np.arange(R, dtype=np.int32)
        row_pos = None
    q_idx, w, q = queries(s, seed, R, layer)
    return Case(s, seed, seq_lens, bt, idx_keys, scales, kv, row_seq, row_pos, q_idx, w, q)


def compact_keys(idx_keys_bf16: np.ndarray):
    """A compact copy of bf16 indexer keys, as a cache would store it next to
    the originals: e4m3 bits of key / scale with one fp32 scale per token
    (its largest magnitude over 448; 1 for an all-zero key).  Returns (bits,
    scales) with the keys' leading shape."""
    import torch
    k = torch.from_numpy(np.ascontiguousarray(idx_keys_bf16).view(np.int16)).view(torch.bfloat16).float().numpy()
    amax = np.abs(k).max(axis=-1)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    return to_e4m3_bits(k / scale[..., None]), scale


def queries(spec: Spec, seed: int, rows: int, layer: int = 0):
    """The query rows of one layer (as make_case draws them): indexer queries
    q_idx [rows, H_I, d_I], weights w [rows, H_I] and attention queries q
    [rows, H, D] (None without a KV cache)."""
    s = spec
    tag = (lambda name: name) if layer == 0 else (lambda name: f"{name}@layer{layer}")
    q_idx = encode(normal((rows, s.n_idx_heads, s.idx_dim), seed, tag("q_idx")), s.act_dtype)
    w = normal((rows, s.n_idx_heads), seed, tag("w"), std=s.w_std)
    q = encode(normal((rows, s.n_heads, s.qk_dim), seed, tag("q")), s.act_dtype) if s.with_kv else None
    return q_idx, w, q


def make_layers(spec: Spec, seed: int, n_layers: int) -> List[Case]:
    """n_layers DSA layers of one decode batch (make_case with layer = 0..n-1)."""
    return [make_case(spec, seed, layer=l) for l in range(n_layers)]


def scaled(spec: Spec, **kw) -> Spec:
    """A smaller workload of the same family (same dtypes and distributions)."""
    return replace(spec, **kw)


def topk_scores(kind: str, rows: int, n: int, seed: int) -> np.ndarray:
    """fp32 score rows for exercising a top-k on fixed inputs.

    kinds: 'normal' (distinct almost surely), 'ties' (few distinct values),
    'equal' (every entry identical), 'signed_zero_inf' (mix of +-0.0, -inf and
    small integers), 'heavy' (lognormal tail), 'neg' (all negative).
    """
    g = rng(seed, "topk_" + kind)
    shape = (rows, n)
    if kind == "normal":
        return normal(shape, seed, "topk_normal")
    if kind == "ties":
        return g.integers(-8, 8, size=shape).astype(np.float32) * np.float32(0.25)
    if kind == "equal":
        return np.full(shape, 1.5, np.float32)
    if kind == "signed_zero_inf":
        choice = g.integers(0, 5, size=shape)
        vals = np.array([0.0, -0.0, -np.inf, 1.0, -1.0], np.float32)
        return vals[choice]
    if kind == "heavy":
        return np.exp(normal(shape, seed, "topk_heavy", std=2.0)).astype(np.float32)
    if kind == "neg":
        return -np.abs(normal(shape, seed, "topk_neg")) - np.float32(1.0)
    raise ValueError(kind)


def index_lists(rows: int, k: int, valid: np.ndarray, seed: int) -> np.ndarray:
    """Sorted ascending distinct positions per row in [0, valid[r]), padded with -1.

    Stands in for a selection when the attention step is exercised on its own.
    """
    g = rng(seed, "index_lists")
    out = np.full((rows, k), -1, np.int32)
    for r in range(rows):
        n = int(min(k, valid[r]))
        if n > 0:
            sel = np.sort(g.choice(int(valid[r]), size=n, replace=False)).astype(np.int32)
            out[r, :n] = sel
    return out


def nbytes_decode_step(case: Case) -> dict:
    """Algorithmic bytes of one decode step, from the drawn lengths.

    keys (+ scales) of every cached token, the block-table entries in use, the
    k gathered KV rows per query row, the queries, weights and outputs.
    """
    s = case.spec
    L = case.seq_lens.astype(np.int64)
    key_b = {"f32": 4, "bf16": 2, "fp8": 1}[s.idx_key_dtype] * s.idx_dim
    act_b = 4 if s.act_dtype == "f32" else 2
    keys = int(L.sum()) * key_b
    scales = int(L.sum()) * 4 if s.idx_key_dtype == "fp8" else 0
    bt = int(((L + s.block_size - 1) // s.block_size).sum()) * 4 if s.block_size else 0
    R = case.rows
    vis = np.minimum(L[case.row_seq], (case.row_pos + 1) if case.row_pos is not None else L[case.row_seq])
    sel = np.minimum(vis, s.top_k)
    gather = int(sel.sum()) * s.qk_dim * act_b
    qi = R * s.n_idx_heads * s.idx_dim * act_b + R * s.n_idx_heads * 4
    q = R * s.n_heads * s.qk_dim * act_b
    out = R * s.n_heads * s.v_dim * act_b
    return {"keys": keys, "scales": scales, "block_table": bt, "kv_gather": gather,
            "q_idx_w": qi, "q": q, "out": out,
            "total": keys + scales + bt + gather + qi + q + out,
            "scores_fp32": int(vis.sum()) * 4}


def flops_prefill_scan(case: Case) -> int:
    s = case.spec
    vis = (case.row_pos.astype(np.int64) + 1) if case.row_pos is not None else case.seq_lens[case.row_seq].astype(np.int64)
    return int(2 * s.n_idx_heads * s.idx_dim * int(vis.sum()))


__all__ = ["Spec", "Case", "WORKLOADS", "workload", "TINY", "DECODE_B1", "DECODE_B32", "DECODE_B4_FP8",
           "PREFILL", "make_case", "make_layers", "queries", "compact_keys", "scaled", "seed_of", "normal", "rng",
           "to_bf16_bits", "to_e4m3_bits", "topk_scores", "index_lists",
           "nbytes_decode_step", "flops_prefill_scan"]
