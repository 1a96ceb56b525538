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


def _run_bench(args, env_extra=None):
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ)
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        env.pop(k, None)
    env.update(env_extra or {})
    p = subprocess.run([sys.executable, os.path.join(root, "bench.py")] + args, cwd=root, env=env,
                       capture_output=True, text=True, timeout=300)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    return [json.loads(l) for l in lines]


def test_reference_arm_prints_one_contract_line():
    """`bench.py --impl reference` times the oracle on the host and prints the same JSON
    line as the library's arm (on a workload small enough for a unit test)."""
    (line,) = _run_bench(["--impl", "reference", "--workload", "tiny_f32_h2_n1024", "--steps", "1",
                          "--warmup", "1"])
    assert line["impl"] == "reference" and line["value"] > 0 and line["higher_is_better"] is True
    assert line["unit"] == "TFLOP/s" and line["config"]["workload"] == "tiny_f32_h2_n1024"
    cpu = line["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] == line["value"] and cpu["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_without_work():
    assert _run_bench(["--impl", "reference", "--workload", "tiny_f32_h2_n1024", "--steps", "1",
                       "--warmup", "1"], {"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"}) == []


def test_clock_summary_from_nvml_samples():
    """The clock record names each throttle reason whose NVML bit was seen and reports the
    median SM clock over the samples taken during the timed region."""
    c = bench.ClockSampler(0)
    c.samples = [(1965.0, 1965.0, 0), (1800.0, 1965.0, 0x4), (1950.0, 1965.0, 0x4 | 0x8)]
    s = c.summary()
    assert s["sm_mhz"] == 1950.0 and s["sm_max_mhz"] == 1965.0 and s["samples"] == 3
    assert s["reasons"] == ["hw_slowdown", "sw_power_cap"]
    assert s["source"].startswith("nvml")
