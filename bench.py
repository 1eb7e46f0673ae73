#!/usr/bin/env python
"""Benchmark of one DSA decode step (indexer scan -> top-k -> sparse MQA) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
    python bench.py --layers 8 --route own|prev --retention R   (several DSA layers per step)

Default workload: batched paged decode, B=32 sequences with lengths drawn
uniformly in [65536, 131072], 64-token blocks under a random block permutation,
a 64-head x 128 bf16 lightning indexer, top-2048, 128-head MQA over 576-wide
bf16 KV rows (value = first 512 columns).  Inputs are seeded synthetic data of
that shape, resident in HBM before timing; the per-step key stream (~805 MB) is
larger than L2, so no explicit flush is needed.

Prints ONE JSON line on rank 0.  With N > 1 (torchrun, one process per GPU) each
rank runs its own independent batch (weak scaling, no collective on the data
path); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from sparse_attention_decode_scan_b200 import synth  # noqa: E402

METRIC = "decode steps/s (scan+top-k+sparse attn) at B=32,128K; % of HBM peak GB/s"
QUERY_SETS = 3  # independently drawn query sets the timed decode steps rotate over
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------------- host-side plumbing

def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def rank_seed(spec, rank: int) -> int:
    """Each rank draws its own batch (independent units, weak scaling)."""
    return synth.seed_of(spec) + 7919 * rank


def reduce_max(x: float, group=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def barrier():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while running."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            if self.thread:
                self.thread.join(timeout=2)

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def source_hash(paths) -> str:
    h = hashlib.sha256()
    for p in paths:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


SCAN_SOURCES = ["sparse_attention_decode_scan_b200/csrc/scan_tc.cuh",
                "sparse_attention_decode_scan_b200/csrc/indexer_tc.cu",
                "sparse_attention_decode_scan_b200/csrc/indexer_simt.cu",
                "sparse_attention_decode_scan_b200/csrc/common.cuh",
                "sparse_attention_decode_scan_b200/csrc/tc.cuh"]


def scan_traffic(workload: str):
    """DRAM bytes per scan launch from the committed ncu summary, if it still
    describes the current scan sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload, {}).get("scan")
    if not e or e.get("source_hash") != source_hash(SCAN_SOURCES):
        return None
    return e.get("dram_bytes_per_launch")


# --------------------------------------------------------------------------- reference arm (the oracle)

def oracle_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_oracle_rate(case, rows, repeats: int = 1):
    """Times the oracle's full step on `rows` (scores, top-k, attention) and
    returns (seconds per row, rows timed)."""
    from oracle import lsa_oracle as O
    t0 = time.perf_counter()
    n = 0
    for _ in range(repeats):
        for r in rows:
            O.row_step(case, r)
            n += 1
    return (time.perf_counter() - t0) / n, n


def run_reference(args, ws_, rank):
    if rank != 0:
        return
    spec = synth.workload(args.workload)
    case = synth.make_case(spec, rank_seed(spec, 0))
    B = case.rows
    per = []
    for i in range(args.warmup + args.steps):
        r = i % B
        t, _ = cpu_oracle_rate(case, [r])
        if i >= args.warmup:
            per.append(t)
    sec_per_step = statistics.mean(per) * B
    value = 1.0 / sec_per_step
    cores = oracle_threads()
    sample = f"{args.steps} timed steps of one sequence each (full scan, top-k, attention), scaled to B={B}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec_per_step * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(case),
            "cpu_baseline": {"value": value, "unit": "steps/s", "cores": cores, "host_cpus": os.cpu_count(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------- our arm

def workload_config(case):
    s = case.spec
    c = {"workload": s.name, "batch": case.rows, "seq_len_min": int(case.seq_lens.min()),
         "seq_len_max": int(case.seq_lens.max()), "seq_len_mean": float(case.seq_lens.mean()),
         "block_size": s.block_size, "idx_heads": s.n_idx_heads, "idx_dim": s.idx_dim,
         "idx_key_dtype": s.idx_key_dtype, "top_k": s.top_k, "heads": s.n_heads, "kv_width": s.qk_dim,
         "v_dim": s.v_dim, "parallelism": "replicas (independent batch per GPU)",
         "query_sets": QUERY_SETS if not s.causal else 1,
         "l2": "inputs larger than L2 (indexer keys streamed from HBM every step)" if s.streams_past_l2
         else "L2 flushed between steps (256 MB write, outside the kernels' event windows)"}
    return c


def run_ours(args, world, rank, local):
    import torch

    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase, to_device

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    base = synth.workload(args.workload)
    spec = base
    if args.batch:
        spec = synth.scaled(spec, batch=args.batch)
    if args.chunk and spec.causal:
        spec = synth.scaled(spec, chunk=args.chunk)
    if args.op == "scan":
        spec = synth.scaled(spec, with_kv=False)
    case = synth.make_case(spec, rank_seed(base, rank))
    dc = DeviceCase(case, device=dev)
    s = case.spec
    R = dc.rows
    ld = (dc.max_len + 3) // 4 * 4
    odt = torch.float32 if s.act_dtype == "f32" else torch.bfloat16
    prefill = s.causal
    scores = torch.empty((R, ld), dtype=torch.float32, device=dev)
    idx = torch.empty((R, s.top_k), dtype=torch.int32, device=dev)
    out = torch.empty((R, s.n_heads, s.v_dim), dtype=odt, device=dev)
    lse = torch.empty((R, s.n_heads), dtype=torch.float32, device=dev)
    ws_bytes = max(lsa.workspace_size(dc.dims, R, dc.max_len, op) for op in
                   (lsa.LSA_OP_SCORES, lsa.LSA_OP_TOPK, lsa.LSA_OP_ATTN, lsa.LSA_OP_DECODE_STEP))
    ws = lsa.workspace(ws_bytes, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = None if base.streams_past_l2 else torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    L = int(case.seq_lens[0])

    run_scan = args.op in ("step", "scan")
    run_topk = args.op in ("step", "topk")
    run_attn = args.op in ("step", "attn")
    if args.op in ("topk", "attn"):  # inputs of the later stages come from one untimed scan (+ top-k)
        lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq,
                           row_pos=dc.row_pos, stream=stream)
        if args.op == "attn":
            lsa.topk(scores, s.top_k, idx, ws, valid_len=None if prefill else dc.seq_lens,
                     n_cols=L if prefill else dc.max_len, ld=ld, stream=stream)

    # The decode step runs through the public one-call entry point (its scan
    # also builds the top-k's first histogram); the profiled variant records
    # the phase-boundary events inside it.
    use_step_api = (not prefill) and args.op == "step"
    step_flags = lsa.LSA_STEP_FUSED if args.fused else lsa.LSA_STEP_UNFUSED
    # Decode steps rotate over QUERY_SETS independently drawn query sets (the
    # case's own plus more draws of the same distributions), so consecutive
    # steps select and gather different KV rows and no step finds the previous
    # one's gathered rows in L2.
    qsets = [(dc.q_idx, dc.w, dc.q)]
    if use_step_api:
        for j in range(1, QUERY_SETS):
            qi, wj, qj = synth.queries(s, rank_seed(base, rank) + 104729 * j, R)
            qsets.append((to_device(qi, s.act_dtype, dev), torch.from_numpy(wj).to(dev),
                          to_device(qj, s.act_dtype, dev)))
    it = [0]

    def step(ev=None):
        if use_step_api:
            qi, wj, qj = qsets[it[0] % len(qsets)]
            it[0] += 1
            if ev is None:
                lsa.decode_step(dc.dims, dc.cache, qi, wj, qj, out, lse, ws, idx_out=idx, flags=step_flags,
                                stream=stream)
            else:
                lsa.decode_step_profiled(dc.dims, dc.cache, qi, wj, qj, out, lse, ws, ev, idx_out=idx,
                                         flags=step_flags, stream=stream)
            return
        if ev is not None:
            ev[0].record(stream)
        if run_scan:
            lsa.indexer_scores(dc.dims, dc.cache, dc.q_idx, dc.w, scores, ld, ws, row_seq=dc.row_seq,
                               row_pos=dc.row_pos, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        if run_topk:
            if prefill:
                lsa.topk(scores, s.top_k, idx, ws, n_cols=L, ld=ld, stream=stream)
            else:
                lsa.topk(scores, s.top_k, idx, ws, valid_len=dc.seq_lens, n_cols=dc.max_len, ld=ld,
                         stream=stream)
        if ev is not None:
            ev[2].record(stream)
        if run_attn:
            lsa.sparse_attn_decode(dc.dims, dc.cache, dc.q, idx, out, lse, ws, row_seq=dc.row_seq,
                                   stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
        if flush is not None:
            flush.zero_()
    torch.cuda.synchronize(dev)
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for e4 in evs:  # create the CUDA events (torch creates them at first record)
        for e in e4:
            e.record(stream)
    torch.cuda.synchronize(dev)
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    with ClockSampler(gpu_index) as clk:
        # keep the GPU under the same load for ~1 s before the timed steps so the
        # clock sampler (100 ms period) sees the loaded state of this workload
        t_soak = time.perf_counter()
        while not args.no_soak and time.perf_counter() - t_soak < 1.0:
            step()
            if flush is not None:
                flush.zero_()
            torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        # Timed region 1 (the value): the plain step, as a caller runs it.  In
        # the decode step the top-k and the attention are programmatic
        # dependents of the kernel before them; events between the kernels
        # would serialise them, so this region records events only around the
        # whole region, or at step boundaries where an L2 flush follows each
        # step (each step's window then excludes the flush).
        bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            # per-step events only where an L2 flush between steps must be left
            # out (each event costs the stream a few microseconds)
            if flush is not None:
                bounds[i][0].record(stream)
            step()
            if flush is not None:
                bounds[i][1].record(stream)
                flush.zero_()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        # Timed region 2 (the breakdown): the same steps with an event at every
        # kernel boundary, for the per-kernel times and the roofline.
        for i in range(args.steps):
            step(evs[i])
            if flush is not None:
                flush.zero_()
        torch.cuda.synchronize(dev)
        barrier()
    total_ms = t_start.elapsed_time(t_end)
    scan_ms = [e[0].elapsed_time(e[1]) for e in evs]
    topk_ms = [e[1].elapsed_time(e[2]) for e in evs]
    attn_ms = [e[2].elapsed_time(e[3]) for e in evs]
    step_ms = [e[0].elapsed_time(e[3]) for e in evs]
    # with a flush between steps the wall window includes it; the step time is the steps' windows
    timed_ms = sum(a.elapsed_time(b) for a, b in bounds) if flush is not None else total_ms
    timed_ms = reduce_max(timed_ms)
    assert lsa.read_device_status(ws) == lsa.LSA_OK

    # e2e: the public decode-step call with host (pinned) inputs and outputs.
    # Every step copies its queries in from pinned host memory and its output
    # and lse back out.  The copies run on their own streams (one per
    # direction) into NBUF rotating device buffers, so step i's output goes
    # out and the queries of steps i+1 .. i+NBUF-1 come in while the next
    # steps compute (a copy gets NBUF-1 steps of time, not one).
    e2e = None
    if not prefill and args.op == "step":
        NBUF = 3
        h_sets = []
        for qi, wj, qj in qsets:
            h_sets.append((qi.cpu().pin_memory(), wj.cpu().pin_memory(), qj.cpu().pin_memory()))
        h_out = [torch.empty(out.shape, dtype=odt).pin_memory() for _ in range(NBUF)]
        h_lse = [torch.empty(lse.shape, dtype=torch.float32).pin_memory() for _ in range(NBUF)]
        d_in = [(torch.empty_like(dc.q_idx), torch.empty_like(dc.w), torch.empty_like(dc.q)) for _ in range(NBUF)]
        d_out = [torch.empty_like(out) for _ in range(NBUF)]
        d_lse = [torch.empty_like(lse) for _ in range(NBUF)]
        s_h2d = torch.cuda.Stream(dev)
        s_d2h = torch.cuda.Stream(dev)

        def e2e_run(n):
            ev_in = [torch.cuda.Event() for _ in range(NBUF)]
            ev_done = [torch.cuda.Event() for _ in range(NBUF)]
            ev_out = [torch.cuda.Event() for _ in range(NBUF)]

            def h2d(i):
                src = h_sets[i % len(h_sets)]
                with torch.cuda.stream(s_h2d):
                    if i >= NBUF:
                        s_h2d.wait_event(ev_done[i % NBUF])  # step i-NBUF has read this buffer
                    for d_t, h_t in zip(d_in[i % NBUF], src):
                        d_t.copy_(h_t, non_blocking=True)
                    ev_in[i % NBUF].record(s_h2d)

            for i in range(min(NBUF, n)):
                h2d(i)
            for i in range(n):
                b = i % NBUF
                stream.wait_event(ev_in[b])
                if i >= NBUF:
                    stream.wait_event(ev_out[b])  # step i-NBUF's output has left this buffer
                qi, wj, qj = d_in[b]
                lsa.decode_step(dc.dims, dc.cache, qi, wj, qj, d_out[b], d_lse[b], ws, flags=step_flags,
                                stream=stream)
                ev_done[b].record(stream)
                with torch.cuda.stream(s_d2h):
                    s_d2h.wait_event(ev_done[b])
                    h_out[b].copy_(d_out[b], non_blocking=True)
                    h_lse[b].copy_(d_lse[b], non_blocking=True)
                    ev_out[b].record(s_d2h)
                if i + NBUF < n:
                    h2d(i + NBUF)
            for b in range(NBUF):
                stream.wait_event(ev_out[b])

        e2e_run(args.warmup)
        torch.cuda.synchronize(dev)
        barrier()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_h2d.wait_stream(stream)
        s_d2h.wait_stream(stream)
        e2e_run(args.steps)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = reduce_max(a.elapsed_time(b_))
        h2d_b = sum(t.numel() * t.element_size() for t in h_sets[0])
        d2h_b = h_out[0].numel() * h_out[0].element_size() + h_lse[0].numel() * 4
        e2e = {"value": world * args.steps / (e2e_ms / 1e3), "unit": "steps/s",
               "h2d_bytes_per_step": int(h2d_b), "d2h_bytes_per_step": int(d2h_b),
               "note": "caches resident in HBM (model state); per-step queries in from pinned host memory and "
                       "output + lse out, on two copy streams through three rotating buffers, overlapped with the neighbouring steps"}

    peaks, peak_src = load_peaks()
    nb = synth.nbytes_decode_step(case)
    ms_per_step = timed_ms / args.steps
    value = world * args.steps / (timed_ms / 1e3)
    scan_avg = statistics.mean(scan_ms)
    # with the fused flag the step is one launch (when it applies): the first
    # phase-event window then holds the whole step
    fused = use_step_api and args.fused and \
        lsa.launch_count(dc.dims, R, dc.max_len, lsa.LSA_OP_DECODE_STEP_FUSED) == 1
    if prefill:
        fl = synth.flops_prefill_scan(case)
        achieved = fl / (scan_avg / 1e3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": scan_traffic(s.name), "kernel": "indexer scan (prefill)",
                "peak_source": f"{peak_src} bf16_tflops (burst)"}
        unit = "chunk rows/s"
        value = world * args.steps * R / (timed_ms / 1e3)
    elif fused:
        # the one launch is the whole step: its algorithmic bytes are the step's
        achieved = nb["total"] / (scan_avg / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": None, "kernel": "fused decode step (scan + top-k + sparse attn, one launch)",
                "algorithmic_bytes_per_launch": nb["total"], "peak_source": f"{peak_src} hbm_gbs"}
        unit = "steps/s"
    else:
        scan_bytes = nb["keys"] + nb["scales"] + nb["block_table"] + nb["q_idx_w"] + nb["scores_fp32"]
        achieved = scan_bytes / (scan_avg / 1e3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": scan_traffic(s.name), "kernel": "indexer scan",
                "algorithmic_bytes_per_launch": scan_bytes, "peak_source": f"{peak_src} hbm_gbs"}
        unit = "steps/s"
    step_gbs = nb["total"] / (ms_per_step / 1e3) / 1e9
    # launches of our kernels per step, as the library plans them for these sizes
    if use_step_api:
        per_step = lsa.launch_count(dc.dims, R, dc.max_len,
                                    lsa.LSA_OP_DECODE_STEP_FUSED if args.fused else lsa.LSA_OP_DECODE_STEP)
    else:
        per_step = sum(lsa.launch_count(dc.dims, R, dc.max_len, op, causal=prefill)
                       for op in (lsa.LSA_OP_SCORES, lsa.LSA_OP_TOPK, lsa.LSA_OP_ATTN)
                       if (op, args.op) in ((lsa.LSA_OP_SCORES, "scan"), (lsa.LSA_OP_TOPK, "topk"),
                                            (lsa.LSA_OP_ATTN, "attn")) or args.op == "step")
    launches = per_step * args.steps

    cpu = None
    if rank == 0 and not args.no_cpu_baseline and s.with_kv:
        sample_rows = [0] if not prefill else [0, R - 1]
        t, n = cpu_oracle_rate(case, sample_rows)
        if prefill:
            cpu_val = 1.0 / t
            cpu_unit = "chunk rows/s"
        else:
            cpu_val = 1.0 / (t * R)
            cpu_unit = "steps/s"
        cpu = {"value": cpu_val, "unit": cpu_unit, "cores": oracle_threads(), "host_cpus": os.cpu_count(),
               "kind": "oracle",
               "sample": f"{n} query row(s) of the same workload through the full oracle step, scaled to the "
                         f"{'chunk' if prefill else 'batch'}"}
    clocks = clk.summary()
    line = {"metric": METRIC if not prefill else "prefill chunk rows/s (causal indexer scan + top-k + sparse attn)",
            "value": value, "unit": unit, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": s.act_dtype if s.idx_key_dtype != "fp8" else "bf16+fp8",
            "data": "synthetic (seeded, generated on host)",
            "config": dict(workload_config(case),
                           step="one cooperative launch (LSA_STEP_FUSED)" if fused else "separate launches"),
            "tokens_per_s": value * R if not prefill else None,
            "step_hbm_gbs": step_gbs, "step_hbm_frac": step_gbs / peaks["hbm_gbs"],
            "step_algorithmic_bytes": nb["total"],
            "kernel_ms": ({"fused_step": scan_avg} if fused else
                          {"scan": scan_avg, "topk": statistics.mean(topk_ms), "attn": statistics.mean(attn_ms)}),
            "kernel_ms_note": "second timed region: events at every kernel boundary (no launch overlap)",
            "ms_per_step_profiled": statistics.mean(step_ms),
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_layers(args, world, rank, local):
    """Several DSA layers per decode step (lsa_decode_layers): the IndexCache
    route (DSA at retention 1) or the MLI route.  Every layer has its own cache
    memory (layer 0's host-drawn cache copied into distinct device buffers, so
    no layer finds another's rows in L2) and its own queries drawn on the host;
    layer l+1 starts after layer l's attention."""
    import torch

    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase, to_device

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    base = synth.workload(args.workload)
    spec = synth.scaled(base, batch=args.batch) if args.batch else base
    assert not spec.causal, "layers: decode workloads only"
    case = synth.make_case(spec, rank_seed(base, rank))
    dc0 = DeviceCase(case, device=dev)
    s = case.spec
    B, n = dc0.rows, args.layers
    route = lsa.LSA_ROUTE_PREV if args.route == "prev" else lsa.LSA_ROUTE_OWN
    caches, q_idx, w, q = [], [], [], []
    keep = []  # device buffers of the layers
    for l in range(n):
        qi, wl, ql = synth.queries(s, rank_seed(base, rank), B, layer=l)
        q_idx.append(to_device(qi, s.act_dtype, dev))
        w.append(torch.from_numpy(wl).to(dev))
        q.append(to_device(ql, s.act_dtype, dev))
        if l == 0:
            caches.append(dc0.cache)
            continue
        keys = dc0.idx_keys.clone()
        scales = dc0.idx_scales.clone() if dc0.idx_scales is not None else None
        kv = dc0.kv.clone()
        keep += [keys, scales, kv]
        c = dc0.make_cache()
        c.idx_keys = keys.data_ptr()
        c.idx_key_scales = scales.data_ptr() if scales is not None else None
        c.kv = kv.data_ptr()
        caches.append(c)
    out = [torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device=dev) for _ in range(n)]
    lse = [torch.empty((B, s.n_heads), dtype=torch.float32, device=dev) for _ in range(n)]
    ws = lsa.workspace(lsa.workspace_size(dc0.dims, B, dc0.max_len, lsa.LSA_OP_DECODE_LAYERS), device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        lsa.decode_layers(dc0.dims, caches, q_idx, w, q, out, lse, ws, retention=args.retention, route=route,
                          stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    with ClockSampler(gpu_index) as clk:
        t_soak = time.perf_counter()
        while not args.no_soak and time.perf_counter() - t_soak < 1.0:
            step()
            torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
    timed_ms = reduce_max(a.elapsed_time(b))
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    peaks, peak_src = load_peaks()
    nb = synth.nbytes_decode_step(case)
    n_ind = len(range(0, n, args.retention))
    # algorithmic bytes: every indexer layer's keys and queries, every layer's gathered rows, query and output
    step_bytes = n_ind * (nb["keys"] + nb["scales"] + nb["block_table"] + nb["q_idx_w"]) + \
        n * (nb["kv_gather"] + nb["q"] + nb["out"])
    ms_per_step = timed_ms / args.steps
    gbs = step_bytes / (ms_per_step / 1e3) / 1e9
    # kernels of the timed steps: a layer with an indexer launches a decode step's, the others an attention's
    launches = args.steps * (n_ind * lsa.launch_count(dc0.dims, B, dc0.max_len, lsa.LSA_OP_DECODE_STEP) +
                             (n - n_ind) * lsa.launch_count(dc0.dims, B, dc0.max_len, lsa.LSA_OP_ATTN))
    route_name = "MLI (previous indexer layer)" if route == lsa.LSA_ROUTE_PREV else \
        ("DSA (own selection)" if args.retention == 1 else "IndexCache (latest indexer layer)")
    line = {"metric": f"decode steps/s over {n} layers, {route_name}, retention 1/{args.retention}",
            "value": world * args.steps / (timed_ms / 1e3), "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "ms_per_layer": ms_per_step / n, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": s.act_dtype if s.idx_key_dtype != "fp8" else "bf16+fp8",
            "data": "synthetic (seeded, generated on host; layer caches are copies of layer 0's in distinct "
                    "device memory, queries drawn per layer)",
            "config": dict(workload_config(case), layers=n, retention=args.retention, route=args.route,
                           indexer_layers=n_ind),
            "step_hbm_gbs": gbs, "step_hbm_frac": gbs / peaks["hbm_gbs"], "step_algorithmic_bytes": step_bytes,
            "peak_source": peak_src, "gpu_launches": launches, "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_two_stage(args, world, rank, local):
    """Decode steps whose selection comes from the two-stage search
    (lsa_two_stage_select: FP8 scan of compact keys, top-n_cand, exact re-score
    of the list with the original keys, top-k) followed by the sparse
    attention.  Reports the selection's bytes and time next to the attention."""
    import torch

    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    base = synth.workload(args.workload)
    spec = synth.scaled(base, batch=args.batch) if args.batch else base
    assert not spec.causal and spec.idx_key_dtype == "bf16", "two-stage: bf16 decode workloads"
    case = synth.make_case(spec, rank_seed(base, rank))
    dc = DeviceCase(case, device=dev)
    bits, scales = synth.compact_keys(case.idx_keys)
    d_bits = torch.from_numpy(np.ascontiguousarray(bits)).to(dev)
    d_scales = torch.from_numpy(scales).to(dev)
    s = case.spec
    B, k, n_cand = dc.rows, s.top_k, args.two_stage
    idx = torch.empty((B, k), dtype=torch.int32, device=dev)
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device=dev)
    ws = lsa.workspace(max(lsa.two_stage_workspace_size(dc.dims, B, dc.max_len, n_cand),
                           lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_ATTN)), device=dev)
    stream = torch.cuda.current_stream(dev)
    qsets = [(dc.q_idx, dc.w, dc.q)]
    for j in range(1, QUERY_SETS):
        qi, wj, qj = synth.queries(s, rank_seed(base, rank) + 104729 * j, B)
        qsets.append((to_dev(qi, s.act_dtype, dev), torch.from_numpy(wj).to(dev), to_dev(qj, s.act_dtype, dev)))

    def step(i, ev=None):
        qi, wj, qj = qsets[i % len(qsets)]
        if ev is not None:
            ev[0].record(stream)
        lsa.two_stage_select(dc.dims, dc.cache, d_bits, d_scales, qi, wj, n_cand, idx, ws, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        lsa.sparse_attn_decode(dc.dims, dc.cache, qj, idx, out, lse, ws, stream=stream)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(dev)
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    gpu_index = int(os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]) \
        if os.environ.get("CUDA_VISIBLE_DEVICES") else local
    with ClockSampler(gpu_index) as clk:
        t_soak = time.perf_counter()
        while not args.no_soak and time.perf_counter() - t_soak < 1.0:
            step(0)
            torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(args.steps):
            step(i)
        b_.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        for i in range(args.steps):
            step(i, evs[i])
        torch.cuda.synchronize(dev)
    timed_ms = reduce_max(a.elapsed_time(b_))
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    sel_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    attn_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    peaks, peak_src = load_peaks()
    nb = synth.nbytes_decode_step(case)
    L = case.seq_lens.astype(np.int64)
    cand_rows = np.minimum(L, n_cand)
    sel_bytes = int(L.sum() * (s.idx_dim + 4) + cand_rows.sum() * s.idx_dim * 2 + nb["block_table"] +
                    nb["q_idx_w"])
    one_stage = int(nb["keys"] + nb["block_table"] + nb["q_idx_w"])
    ms_per_step = timed_ms / args.steps
    line = {"metric": f"decode steps/s with the two-stage selection (list of {n_cand}) + sparse attn",
            "value": world * args.steps / (timed_ms / 1e3), "unit": "steps/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16+fp8", "data": "synthetic (seeded)",
            "config": dict(workload_config(case), n_cand=n_cand),
            "kernel_ms": {"two_stage_select": sel_ms, "attn": attn_ms},
            "selection_algorithmic_bytes": sel_bytes, "one_stage_scan_bytes": one_stage,
            "selection_bytes_ratio": sel_bytes / one_stage,
            "selection_hbm_frac": sel_bytes / (sel_ms / 1e3) / 1e9 / peaks["hbm_gbs"],
            "peak_source": peak_src, "gpu_launches": args.steps * 8, "clocks": clk.summary()}
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_blocks(args, world, rank, local):
    """Layers that attend whole KV blocks picked a layer ahead, with the KV cache
    offloaded to page-locked host memory (SparDA abstract: a forecast of the
    next layer's blocks lets their host-to-device copy overlap the current
    layer).  Per layer l, on the compute stream: the next layer's indexer scan
    and block selection (lsa_block_select), then layer l's sparse attention
    over its staged blocks; on a copy stream, concurrently: the next layer's
    kept blocks copied from host memory into the other staging buffer
    (lsa_stage_blocks).  The forecast query of layer l+1 is that layer's own
    indexer query (the trained Forecast projection is out of scope).  Also
    times the same layers with the copy in line (no overlap)."""
    import torch

    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase, make_dims

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    base = synth.workload(args.workload)
    spec = synth.scaled(base, batch=args.batch) if args.batch else base
    assert not spec.causal and spec.block_size > 0, "blocks: paged decode workloads"
    case = synth.make_case(spec, rank_seed(base, rank))
    dc = DeviceCase(case, device=dev)
    s = case.spec
    B, bs, n_sel = dc.rows, s.block_size, args.blocks
    n_layers = args.layers if args.layers > 1 else 4
    host_kv = dc.kv.cpu().pin_memory()  # the offloaded KV cache (one copy serves every layer)
    hcache = dc.make_cache()
    hcache.kv = host_kv.data_ptr()
    qs = []
    for l in range(n_layers + 1):
        qi, wl, ql = synth.queries(s, rank_seed(base, rank), B, layer=l)
        qs.append((to_dev(qi, s.act_dtype, dev), torch.from_numpy(wl).to(dev), to_dev(ql, s.act_dtype, dev)))
    ld = (dc.max_len + 3) // 4 * 4
    scores = torch.empty((B, ld), dtype=torch.float32, device=dev)
    kept = [torch.empty((B, n_sel), dtype=torch.int32, device=dev) for _ in range(2)]
    staged = [torch.empty((B * n_sel, bs, s.qk_dim), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    table = [torch.empty((B, n_sel), dtype=torch.int32, device=dev) for _ in range(2)]
    sidx = [torch.empty((B, n_sel * bs), dtype=torch.int32, device=dev) for _ in range(2)]
    lens = torch.full((B,), n_sel * bs, dtype=torch.int32, device=dev)
    scache = [lsa.staged_cache(staged[i], table[i], lens, n_sel, bs) for i in range(2)]
    ad = make_dims(s, top_k=n_sel * bs)
    out = torch.empty((B, s.n_heads, s.v_dim), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, s.n_heads), dtype=torch.float32, device=dev)
    ws_c = lsa.workspace(max(lsa.workspace_size(dc.dims, B, dc.max_len, lsa.LSA_OP_SCORES),
                             lsa.block_select_workspace_size(B, dc.max_len, bs, n_sel),
                             lsa.workspace_size(ad, B, n_sel * bs, lsa.LSA_OP_ATTN)), device=dev)
    ws_x = lsa.workspace(256, device=dev)
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)

    def select(l):
        qi, wl, _ = qs[l]
        lsa.indexer_scores(dc.dims, dc.cache, qi, wl, scores, ld, ws_c, stream=comp)
        lsa.block_select(scores, bs, n_sel, kept[l % 2], ws_c, valid_len=dc.seq_lens, n_cols=dc.max_len, ld=ld,
                         stream=comp)

    def stage(l, st):
        lsa.stage_blocks(dc.dims, hcache, kept[l % 2], bs, staged[l % 2], table[l % 2], sidx[l % 2], ws_x, stream=st)

    def attend(l):
        lsa.sparse_attn_decode(ad, scache[l % 2], qs[l][2], sidx[l % 2], out, lse, ws_c, stream=comp)

    def step(overlap):
        select(0)
        stage(0, comp)
        for l in range(n_layers):
            if l + 1 < n_layers:
                select(l + 1)  # the forecast of the next layer's blocks
                ev = torch.cuda.Event()
                ev.record(comp)
                st = copy if overlap else comp
                if overlap:
                    copy.wait_event(ev)
                stage(l + 1, st)
                done = torch.cuda.Event()
                done.record(st)
            attend(l)
            if l + 1 < n_layers:
                comp.wait_event(done)

    res = {}
    for overlap in (True, False):
        for _ in range(args.warmup):
            step(overlap)
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(comp)
        for _ in range(args.steps):
            step(overlap)
        b_.record(comp)
        torch.cuda.synchronize(dev)
        res[overlap] = reduce_max(a.elapsed_time(b_)) / args.steps
    assert lsa.read_device_status(ws_c) == lsa.LSA_OK and lsa.read_device_status(ws_x) == lsa.LSA_OK
    # the host link's copy rate for reference: one large page-locked copy
    probe = torch.empty(256 << 20, dtype=torch.uint8).pin_memory()
    dprobe = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    dprobe.copy_(probe, non_blocking=True)
    a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    for _ in range(4):
        dprobe.copy_(probe, non_blocking=True)
    b_.record(comp)
    torch.cuda.synchronize(dev)
    h2d_gbs = 4 * probe.numel() / (a.elapsed_time(b_) / 1e3) / 1e9
    L = case.seq_lens.astype(np.int64)
    staged_bytes = int(np.minimum((L + bs - 1) // bs, n_sel).sum()) * bs * s.qk_dim * 2
    ms = res[True]
    line = {"metric": f"decode steps/s over {n_layers} layers attending {n_sel} KV blocks each, blocks of the next "
                      f"layer staged from host memory during the current one",
            "value": world / (ms / 1e3), "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "ms_per_step_copy_in_line": res[False],
            "overlap_gain": res[False] / ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic (seeded); KV in page-locked host memory",
            "config": dict(workload_config(case), layers=n_layers, n_sel=n_sel, block_size=bs),
            "staged_bytes_per_layer": staged_bytes,
            "host_link_gbs_achieved": staged_bytes * (n_layers) / (ms / 1e3) / 1e9,
            "host_link_gbs_plain_copy": h2d_gbs,
            # per layer: scan, block maximum, top-k (histogram + select), staging copy, attention
            "gpu_launches": args.steps * n_layers * 6,
            }
    if rank == 0:
        print(json.dumps(line), flush=True)


def run_prefill_layers(args, world, rank, local):
    """The prefill workload through several layers (lsa_prefill_layers), each
    layer's history (131072 KV rows) in page-locked host memory and streamed
    through two alternating device buffers, rows in blocks of --row-block.
    Every layer uses layer 0's data (one host copy of the history; the copy
    and the compute are what is timed).  Also times the same layers with the
    history already on the device (no copy), for the overlap."""
    import torch

    from sparse_attention_decode_scan_b200 import lsa
    from sparse_attention_decode_scan_b200.device import DeviceCase

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    base = synth.workload(args.workload)
    if not base.causal:  # the mode runs the causal prefill workload
        base = synth.workload(synth.PREFILL)
    spec = synth.scaled(base, chunk=args.chunk) if args.chunk else base
    case = synth.make_case(spec, rank_seed(base, rank))
    dc = DeviceCase(case, device=dev)
    s = case.spec
    R, L = dc.rows, dc.max_len
    n = args.layers if args.layers > 1 else 3
    hist_len = int(case.row_pos[0])
    host_hist = dc.kv[0, :hist_len].cpu().pin_memory()
    dev_hist = dc.kv[0, :hist_len].contiguous()
    chunk = dc.kv[0, hist_len:L].contiguous()
    outs = [torch.empty((R, s.n_heads, s.v_dim), dtype=torch.bfloat16, device=dev) for _ in range(n)]
    bufs = [torch.empty((L, s.qk_dim), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    rb = args.row_block if args.row_block else R
    ws = lsa.workspace(lsa.prefill_layers_workspace_size(dc.dims, R, L, rb), device=dev)
    events = [torch.cuda.Event() for _ in range(4)]
    copy = torch.cuda.Stream(dev)
    comp = torch.cuda.current_stream(dev)

    def run(hist):
        caches = []
        for _ in range(n):
            c = dc.make_cache()
            c.kv = hist.data_ptr()
            caches.append(c)
        lsa.prefill_layers(dc.dims, caches, hist_len, [chunk] * n, dc.row_pos, [dc.q_idx] * n, [dc.w] * n,
                           [dc.q] * n, outs, None, bufs, ws, rb, events, stream=comp, copy_stream=copy)

    res = {}
    for name, hist in (("host", host_hist), ("device", dev_hist)):
        for _ in range(args.warmup):
            run(hist)
        torch.cuda.synchronize(dev)
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(comp)
        for _ in range(args.steps):
            run(hist)
        b_.record(comp)
        torch.cuda.synchronize(dev)
        res[name] = reduce_max(a.elapsed_time(b_)) / args.steps
    assert lsa.read_device_status(ws) == lsa.LSA_OK
    ms = res["host"]
    kv_row = s.qk_dim * 2
    line = {"metric": f"prefill chunk rows/s through {n} layers, history streamed from host memory through two "
                      f"device buffers", "value": world * R * n / (ms / 1e3), "unit": "chunk rows x layers / s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_layer": ms / n, "ms_per_step_history_on_device": res["device"],
            "copy_hidden_frac": res["device"] / ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded); history in page-locked host memory",
            "config": dict(workload_config(case), layers=n, row_block=rb, history_rows=hist_len),
            "history_bytes_per_layer": hist_len * kv_row,
            "device_history_bytes": 2 * L * kv_row, "device_history_bytes_all_layers_resident": n * L * kv_row,
            "score_workspace_bytes": rb * ((L + 3) // 4 * 4) * 4,
            "score_workspace_bytes_unblocked": R * ((L + 3) // 4 * 4) * 4,
            "gpu_launches": args.steps * n * ((R + rb - 1) // rb) * 4}
    if rank == 0:
        print(json.dumps(line), flush=True)


def to_dev(arr, dtype, dev):
    from sparse_attention_decode_scan_b200.device import to_device
    return to_device(arr, dtype, dev)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=synth.DECODE_B32,
                    help="workload name (or a unique prefix of one): " + ", ".join(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    # profiling aids: a smaller batch of the same workload, one stage only, no clock soak
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling)")
    ap.add_argument("--chunk", type=int, default=0,
                    help="prefill: the last CHUNK rows of the workload's chunk only (profiling)")
    ap.add_argument("--op", default="step", choices=["step", "scan", "topk", "attn"],
                    help="time one stage only (profiling); the bench line is for 'step'")
    ap.add_argument("--no-soak", action="store_true", help="skip the 1 s clock-sampling soak (profiling)")
    ap.add_argument("--layers", type=int, default=1,
                    help="DSA layers per decode step (lsa_decode_layers); 1 = the single-layer step")
    ap.add_argument("--route", default="own", choices=["own", "prev"],
                    help="layers: attend the latest indexer layer at or before (own) or before (prev, MLI) a layer")
    ap.add_argument("--retention", type=int, default=1, help="layers: every retention-th layer keeps an indexer")
    ap.add_argument("--prefill-layers", action="store_true",
                    help="the prefill workload through --layers layers, history streamed from host memory")
    ap.add_argument("--row-block", type=int, default=0, help="prefill layers: query rows per block (0: all)")
    ap.add_argument("--blocks", type=int, default=0, metavar="N_SEL",
                    help="layers attending N_SEL KV blocks each, staged from host memory a layer ahead")
    ap.add_argument("--two-stage", type=int, default=0, metavar="N_CAND",
                    help="decode steps whose selection is the two-stage search with a list of N_CAND")
    ap.add_argument("--fused", action="store_true",
                    help="decode step as one cooperative launch (LSA_STEP_FUSED) instead of separate launches")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_env()
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            if args.two_stage:
                run_two_stage(args, world, rank, local)
            elif args.blocks:
                run_blocks(args, world, rank, local)
            elif args.prefill_layers:
                run_prefill_layers(args, world, rank, local)
            elif args.layers > 1:
                run_layers(args, world, rank, local)
            else:
                run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
