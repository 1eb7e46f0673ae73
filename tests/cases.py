"""Workloads of the parity tests: scaled-down members of each benchmark family
(several tiles plus a ragged tail, oracle-sized) and the full-size shapes."""
import functools

from sparse_attention_decode_scan_b200 import synth

W = synth.WORKLOADS

SMALL = {
    # full tiny fp32 workload
    "tiny_fp32": W[synth.TINY],
    # production widths, one sequence of a length that is not a multiple of 128
    "bf16_L5000": synth.scaled(W[synth.DECODE_B1], len_lo=5000, len_hi=5000),
    # paged batch with lengths below and above k (-1 padding and ragged tails)
    "paged_B5": synth.scaled(W[synth.DECODE_B32], batch=5, len_lo=100, len_hi=4000, top_k=512),
    # FP8 keys with the heavy-tailed dimension, ragged length
    "fp8_L6001": synth.scaled(W[synth.DECODE_B4_FP8], batch=2, len_lo=6001, len_hi=6001),
    # causal prefill chunk of 256 rows over 3000 tokens
    "prefill_3000x256": synth.scaled(W[synth.PREFILL], len_lo=3000, len_hi=3000, chunk=256, top_k=512),
    # single short sequence (length 1) and contiguous bf16
    "len1": synth.scaled(W[synth.DECODE_B1], batch=3, len_lo=1, len_hi=300, top_k=64),
    # pages of 48 tokens (not a power of two; the tensor-core scan takes multiples of 64, so its
    # scan runs on the CUDA cores)
    "paged48_B3": synth.scaled(W[synth.DECODE_B32], batch=3, len_lo=300, len_hi=2500, top_k=256, block_size=48),
}

SEEDS = {name: 5000 + i for i, name in enumerate(SMALL)}


@functools.lru_cache(maxsize=None)
def small(name: str):
    return synth.make_case(SMALL[name], SEEDS[name])


def full(name: str, with_kv: bool = True):
    """A full-size workload (its own seed)."""
    spec = W[name] if with_kv else synth.scaled(W[name], with_kv=False)
    return synth.make_case(spec, synth.seed_of(spec))
