"""Host-side logic of the N>1 bench path on CPU: two gloo ranks.

The data path has no collective (each rank runs an independent batch); the only
cross-rank steps are the barrier around the timed region and the max-over-ranks
reduction of the elapsed time.  Ranks draw different batches.
"""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier()
        elapsed = 10.0 + 5.0 * rank       # rank 1 is the slow one
        m = bench.reduce_max(elapsed)
        ws, rk, lr = bench.dist_env()
        q.put((rank, m, bench.rank_seed(bench.synth.WORKLOADS[bench.synth.DECODE_B32], rank), ws, rk))
        bench.barrier()
    finally:
        dist.destroy_process_group()


def test_two_ranks_max_time_and_distinct_batches():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    assert [r[1] for r in res] == [15.0, 15.0]          # both ranks see the slowest time
    assert res[0][2] != res[1][2]                       # independent batches
    assert [r[3] for r in res] == [2, 2] and [r[4] for r in res] == [0, 1]


def test_reference_arm_prints_on_rank0_only(capsys):
    import argparse

    import bench
    args = argparse.Namespace(workload=bench.synth.TINY, steps=1, warmup=3, gpus=2)
    bench.run_reference(args, 2, 1)                     # rank 1: no work, no output
    assert capsys.readouterr().out == ""


def test_single_process_reduce_is_identity():
    import bench
    assert bench.reduce_max(3.5) == 3.5
