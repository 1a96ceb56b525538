"""Host logic of bench.py's multi-GPU replica path, on CPU: two gloo ranks.

Each rank is an independent replica (no data-path collective); the job's time is the slowest
rank's, taken with an all-reduce MAX, and the reported value aggregates all ranks' work over
that time.  Only the timing reduction and the barriers are collective.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, ws: int, port: int, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(ws), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        e_ws, e_rank, e_local = bench.dist_env()
        bench.barrier(ws)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, ws)   # rank 1 is the slow one
        bench.barrier(ws)
        out.put((e_ws, e_rank, e_local, t))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_over_ranks_and_env():
    ws, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, ws, port, q)) for r in range(ws)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(ws))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [(r[0], r[1], r[2]) for r in res] == [(2, 0, 0), (2, 1, 1)]
    assert all(r[3] == 15.0 for r in res)          # every rank sees the slowest time


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)


def test_aggregate_counts_every_replica():
    # 2 replicas of 3.554 TFLOP each in 10 ms (the slowest rank) -> 710.8 TFLOP/s
    assert bench.aggregate_tflops(3_554_000_000_000, 10.0, 2) == pytest.approx(710.8)
    assert bench.aggregate_tflops(3_554_000_000_000, 10.0, 1) == pytest.approx(355.4)
