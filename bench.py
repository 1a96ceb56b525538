"""Benchmark of the RoLA attention forward on B200.

One step = one whole forward pass (block pooling + top-k selection, linear state,
sparse attention with the fused linear epilogue) over the Wan2.1-14B-720P-shaped
workload (B=1, H=40, N=75600 = 21x45x80, d=128, r=32, topk=0.03, bf16) with the
inputs resident in HBM.  The metric is kept-block TFLOP/s: the algorithmic FLOPs of
the sparse branch, 4*d*c_i*c_j summed over every kept (query block i, key block j)
pair (c = valid tokens of a block), divided by the step time.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl rola|reference]
                  [--gate head|token] [--no-e2e] [--no-cpu-baseline] [--no-fp8] [--no-backward]

``--gate token`` feeds a gain per token and head (g [B, N, H]) instead of per head;
``--gate proj`` has the library compute it from the query (gate_proj, gate_bias).
For a bf16 workload that has an fp8-e4m3 twin (the 720P and 480P 14B shapes), the same
line also carries ``fp8``: the twin timed the same way on the same inputs (``--no-fp8``
skips it).  ``backward`` times rola_backward (the gradients of the same forward, fp32
gradients) on the same workload: a few calls, the same timing rules; its TFLOP/s counts the
five kept-block products of an attention backward (2.5 x the forward's kept-block FLOPs).

Multi-GPU (torchrun, one rank per GPU): every rank runs an independent forward of the
same workload (different seed), no collective on the data path ("scaling": "weak");
the time is the max over ranks.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload on rank 0.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "RoLA fwd kept-block TFLOP/s at Wan2.1-14B-720P shape, 1xB200"
UNIT = "TFLOP/s"


# key/value pass, state reduction | query pass | block scores, top-k | attention fast and
# careful passes
LAUNCHES_PER_STEP = 7

# DRAM bytes (read + write) per launch of the attention kernel's fast pass, from
# `dram__bytes_read.sum + dram__bytes_write.sum` of one ncu capture of the current kernel on the
# 14B-480P workload, scaled to 720P by the token count (the streamed bytes grow with N).  None
# where no capture of the current kernel exists.
ATTEND_DRAM_BYTES = {"wan21_14b_720p": 1.510e9 * 75600 / 32760, "wan21_14b_480p": 1.510e9,
                     "wan21_14b_720p_fp8": 0.9972e9 * 75600 / 32760, "wan21_14b_480p_fp8": 0.9972e9}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kept_block_flops(col: torch.Tensor, N: int, d: int) -> int:
    """4*d*c_i*c_j over every kept pair; col is [B, H, nb, k] int32 on the device."""
    B, H, nb, k = col.shape
    c = torch.full((nb,), 64, dtype=torch.int64, device=col.device)
    c[-1] = N - 64 * (nb - 1)
    kept = c[col.long()].sum(-1)                 # [B, H, nb] sum_j c_j
    return int((kept * c.view(1, 1, nb)).sum().item()) * 4 * d


def linear_epilogue_flops(w) -> int:
    """Query-side linear branch inside the attention kernel: u = q Wq and num = (R u) S."""
    return 4 * w.B * w.H * w.N * w.d * w.r


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons sampled during the timed region, every
    10 ms through NVML (the GPU found by its PCI bus id, so CUDA_VISIBLE_DEVICES does not
    matter); ``nvidia-smi -lms 100`` when NVML is not usable."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap"}

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.dev = device_index
        self.period = period_s
        self.proc = None
        self.thread = None
        self.samples = []       # (sm_mhz, max_mhz, reason bits)
        self.lines = []

    def _bus_id(self):
        p = torch.cuda.get_device_properties(self.dev)
        return f"{p.pci_domain_id:08x}:{p.pci_bus_id:02x}:{p.pci_device_id:02x}.0"

    def _nvml_loop(self, nv, h):
        import threading
        while not self._stop.is_set():
            try:
                sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            self._stop.wait(self.period)

    def __enter__(self):
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            try:
                h = nv.nvmlDeviceGetHandleByPciBusId(self._bus_id().encode())
            except Exception:
                h = nv.nvmlDeviceGetHandleByIndex(self.dev)
            self._nv = nv
            self._stop = threading.Event()
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, h), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self._bus_id()}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.thread is not None:
            self._stop.set()
            self.thread.join(timeout=5)
            try:
                self._nv.nvmlShutdown()
            except Exception:
                pass
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        for s_mhz, m_mhz, bits in self.samples:
            sm.append(s_mhz)
            mx = m_mhz
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvml, 10 ms" if self.samples else "nvidia-smi, 100 ms"}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def max_over_ranks(x: float, ws: int) -> float:
    """Largest value of x over the ranks (the job's time is its slowest rank's)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(flops_per_rank: int, ms_per_step_max: float, ws: int) -> float:
    """Whole-job throughput of ws independent replicas: all ranks' work over the slowest time."""
    return ws * flops_per_rank / (ms_per_step_max * 1e-3) / 1e12


def barrier(ws: int):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle baseline

def oracle_sample(w, seconds_hint=15.0, seed=0):
    """Times the oracle as it stands on a bounded sample of workload ``w``, about
    ``seconds_hint`` of CPU time: head after head (each with its full pooling, selection
    and linear state), attention on a seeded set of query blocks that grows to the time
    left; each head's time is extrapolated to all its query blocks."""
    import numpy as np
    import oracle as O
    start = time.perf_counter()
    t_sum = flops_sum = 0.0
    heads = blocks_run = 0
    for hh in range(w.H):
        sub = synth.custom(w.name + "_sample", B=1, H=1, N=w.N, d=w.d, r=w.r, topk=w.topk,
                           grid=w.grid, dtype=w.dtype, dist=w.dist)
        inp = synth.make_inputs(sub, seed=1000 * seed + hh, device="cpu")
        h = {k: v.float().numpy() for k, v in inp.items()}
        s = O.make_shape(1, 1, sub.N, sub.d, sub.r, sub.topk, grid=sub.grid)
        t0 = time.perf_counter()
        qbar, kbar = O.pool(s, h["q"]), O.pool(s, h["k"])
        col, *_ = O.select(s, qbar, kbar)
        S, z = O.linear_state(s, h["k"], h["v"], h["Wk"])
        t_pre = time.perf_counter() - t0
        order = np.random.default_rng(seed + hh).permutation(w.nb)
        n0 = max(8, min(w.nb, int(8 * O.threads())))

        def run(sel):
            blocks = np.array([(0, 0, i) for i in sorted(sel)], dtype=np.int32)
            t = time.perf_counter()
            O.attend_blocks(s, h["q"], h["k"], h["v"], h["Wq"], h["g"], col, S, z, blocks)
            return time.perf_counter() - t

        t_att = run(order[:n0].tolist())
        left = seconds_hint - (time.perf_counter() - start)
        n_more = max(0, min(w.nb - n0, int(left / (t_att / n0))))
        if n_more > 0:
            t_att += run(order[n0:n0 + n_more].tolist())
        n = n0 + n_more
        t_sum += t_pre + t_att * (w.nb / n)
        c = np.full(w.nb, 64, dtype=np.int64)
        c[-1] = w.N - 64 * (w.nb - 1)
        flops_sum += 4 * w.d * int((c[col[0, 0]].sum(-1) * c).sum())
        heads += 1
        blocks_run += n
        elapsed = time.perf_counter() - start
        if elapsed >= 0.8 * seconds_hint or elapsed + t_pre + t_att * (w.nb / n) > 1.5 * seconds_hint:
            break
    return {"value": flops_sum / t_sum / 1e12, "seconds": time.perf_counter() - start,
            "cores": O.threads(),
            "sample": (f"{heads} of {w.H} heads, each with its full pooling, block selection and "
                       f"linear state; sparse+linear attention on {blocks_run} of {heads * w.nb} "
                       f"query blocks, each head's time extrapolated to all its blocks")}


# ------------------------------------------------------------------ device timing

def measure(w, plan, step, steps, warmup, ws, dev):
    """Times exactly ``steps`` calls of ``step`` (after ``warmup`` untimed ones) with CUDA
    events on the launching stream, bracketed by a barrier and a synchronize on both
    sides; the time is the max over ranks.  Stage times come from the library's own
    events between the forward's stages, recorded in the same timed calls."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    assert plan.poll_status() == 0
    flops = kept_block_flops(plan.block_lists(), w.N, w.d)
    plan.profile_stages(True)      # events between the forward's stages (host call, untimed)
    barrier(ws)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for _ in range(steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
    barrier(ws)
    ms_total = max_over_ranks(t0.elapsed_time(t1), ws)
    stage_sum, ncalls = plan.stage_times()
    plan.profile_stages(False)
    assert plan.poll_status() == 0
    return {"flops": flops, "ms_step": ms_total / steps,
            "stage_ms": [x / ncalls for x in stage_sum] if ncalls else None,
            "clocks": clk.summary()}


def roofline(w, stage_ms, flops):
    """The attention kernel (kept-block + linear-epilogue FLOPs over its stage time) against
    the measured dense tensor peak of its operand type: the sustained figure (cuBLAS in a
    seconds-long loop), since the kernel is timed inside the long timed region; the burst
    figure's fraction rides along."""
    peaks = load_peaks()
    att_ms = stage_ms[-1]
    achieved = (flops + linear_epilogue_flops(w)) / (att_ms * 1e-3) / 1e12
    ratio = 2.0 if w.dtype == "fp8" else 1.0   # e4m3 products: the bf16 figure x nominal 4.5 / 2.25
    peak = ratio * peaks["bf16_tflops_sustained"]
    burst = ratio * peaks["bf16_tflops"]
    what = " x 2 (nominal fp8/bf16 ratio)" if w.dtype == "fp8" else ""
    return {"bound": "tensor", "kernel": "attend (sparse branch + fused linear epilogue)",
            "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": ATTEND_DRAM_BYTES.get(w.name), "traffic_unit": "bytes/launch",
            "peak_source": f"{peaks['source']} bf16 sustained (cuBLAS 8192^3 back to back for 4 s){what}",
            "peak_burst": burst, "frac_burst": achieved / burst}


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="wan21_14b_720p")
    ap.add_argument("--impl", default="rola", choices=["rola", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-fp8", action="store_true", help="skip the fp8-e4m3 twin of a bf16 workload")
    ap.add_argument("--no-backward", action="store_true", help="skip the backward measurement")
    ap.add_argument("--gate", default="head", choices=["head", "token", "proj"],
                    help="gain of the linear branch per head (default), per token and head, or "
                         "computed from the query (sigmoid of q . gate_proj + gate_bias)")
    args = ap.parse_args()
    ws, rank, local = dist_env()
    w = synth.WORKLOADS[args.workload]

    if args.impl == "reference":
        if rank != 0:
            return
        vals = []
        samp = None
        for it in range(args.warmup + args.steps):
            r = oracle_sample(w, seconds_hint=max(0.5, 150.0 / (args.warmup + args.steps)), seed=it)
            if it >= args.warmup:
                vals.append(r["value"])
                samp = r
        v = statistics.median(vals)
        line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": None,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N,
                                                "d": w.d, "r": w.r, "topk": w.topk},
                "cpu_baseline": {"value": v, "unit": UNIT, "cores": samp["cores"], "kind": "oracle",
                                 "sample": samp["sample"]},
                "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import sparse_rank_attention_b200 as rola
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    rola.load()
    inp = synth.make_inputs(w, seed=rank, device=dev)
    per_token = args.gate != "head"
    if args.gate == "token":
        inp["g"] = synth.make_gate(w, seed=100 + rank, device=dev)        # [B, N, H]
    elif args.gate == "proj":
        inp["g"] = synth.make_gate_proj(w, seed=100 + rank, device=dev)   # [H*(d+1)]
    plan = rola.Plan.for_workload(w, device=dev, gate=args.gate)
    out = torch.empty_like(inp["q"])
    q, k, v, Wq, Wk, g = (inp[x] for x in ("q", "k", "v", "Wq", "Wk", "g"))
    stream = torch.cuda.current_stream()

    def step():
        plan.forward(q, k, v, Wq, Wk, g, out)

    m = measure(w, plan, step, args.steps, args.warmup, ws, dev)
    flops, ms_step, stage_ms, clk = m["flops"], m["ms_step"], m["stage_ms"], m["clocks"]
    value = aggregate_tflops(flops, ms_step, ws)
    roof = roofline(w, stage_ms, flops)
    act = w.B * w.N * w.H * w.d                     # elements of one activation tensor
    nblk = w.B * w.H * plan.nb
    if len(stage_ms) == 4:
        # HBM bytes of the two passes.  The method's own bytes: each pass reads its inputs
        # once (k and v; q).  The build's intermediates on top: the fp16 copy of v (bf16) or
        # the e4m3 k and v (fp8) written by the key/value pass; the query-feature images,
        # g/den, the q means (and e4m3 q) written by the query pass.
        kv_method, q_method = 2 * act * 2, act * 2
        kv_extra = 2 * act if w.dtype == "fp8" else act * 2
        q_extra = nblk * (2 * w.r * 128 + 64 * 4 + w.d * 4) + (act if w.dtype == "fp8" else 0)
        stages = {"kv_pass_ms": stage_ms[0], "query_pass_ms": stage_ms[1], "select_ms": stage_ms[2],
                  "attend_ms": stage_ms[3],
                  "pre_attention_ms": stage_ms[0] + stage_ms[1] + stage_ms[2],
                  "kv_pass_GBs_method": kv_method / (stage_ms[0] * 1e-3) / 1e9,
                  "query_pass_GBs_method": q_method / (stage_ms[1] * 1e-3) / 1e9,
                  "passes_frac_hbm_method": (kv_method + q_method) / ((stage_ms[0] + stage_ms[1]) * 1e-3) / 1e9
                  / load_peaks()["hbm_gbs"],
                  "kv_pass_GBs_with_copies": (kv_method + kv_extra) / (stage_ms[0] * 1e-3) / 1e9,
                  "query_pass_GBs_with_copies": (q_method + q_extra) / (stage_ms[1] * 1e-3) / 1e9}
    else:
        stages = {"select_blocks_ms": stage_ms[0], "linear_state_ms": stage_ms[1], "attend_ms": stage_ms[2]}

    e2e = None
    if not args.no_e2e:
        # End to end through the public call with host-resident inputs, pipelined the way a
        # serving loop is: step n's inputs are copied in (pinned host -> device, copy stream)
        # while step n - 1 computes, and step n - 1's output is copied back (device -> pinned
        # host, a third stream) while step n computes.  Every step moves all its own bytes;
        # device inputs and outputs are double-buffered.
        hq, hk, hv = (x.cpu().pin_memory() for x in (q, k, v))
        hWq, hWk, hg = (x.cpu().pin_memory() for x in (Wq, Wk, g))
        hsrc = (hq, hk, hv, hWq, hWk, hg)
        hout = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        dset = [tuple(torch.empty_like(x) for x in (q, k, v, Wq, Wk, g)) for _ in range(2)]
        dout = [torch.empty_like(out) for _ in range(2)]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_cmp = stream
        ev = {n: [torch.cuda.Event() for _ in range(2)] for n in ("in", "cmp", "out")}
        issued = [0]

        def e2e_step():
            n = issued[0]
            sl = n % 2
            if n >= 2:
                s_in.wait_event(ev["cmp"][sl])        # the forward two steps back read this set
            with torch.cuda.stream(s_in):
                for dst, src in zip(dset[sl], hsrc):
                    dst.copy_(src, non_blocking=True)
                ev["in"][sl].record(s_in)
            s_cmp.wait_event(ev["in"][sl])
            if n >= 2:
                s_cmp.wait_event(ev["out"][sl])       # its output buffer has been copied back
            plan.forward(*dset[sl], dout[sl], stream=s_cmp)
            ev["cmp"][sl].record(s_cmp)
            s_out.wait_event(ev["cmp"][sl])
            with torch.cuda.stream(s_out):
                hout[sl].copy_(dout[sl], non_blocking=True)
                ev["out"][sl].record(s_out)
            issued[0] += 1

        e_steps = max(20, min(args.steps, 40))
        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize()
        barrier(ws)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s_in)
        for _ in range(e_steps):
            e2e_step()
        b.record(s_out)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(a.elapsed_time(b), ws) / e_steps
        h2d = sum(x.numel() * x.element_size() for x in hsrc)
        e2e = {"value": aggregate_tflops(flops, e_ms, ws), "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": hout[0].numel() * hout[0].element_size(),
               "pipelined": "inputs of step n copied in while step n-1 computes; outputs copied back "
                            "while the next step computes (3 streams, double-buffered device tensors)"}
        assert plan.poll_status() == 0

    fp8 = None
    twin = synth.WORKLOADS.get(w.name + "_fp8")
    if twin is not None and w.dtype == "bf16" and not args.no_fp8:
        # the fp8-e4m3 twin on the same bf16 inputs: quantised inside the call, so the
        # same step and the same timing rules; kept-block FLOPs are the same
        plan8 = rola.Plan.for_workload(twin, device=dev, gate=args.gate)
        out8 = torch.empty_like(out)

        def step8():
            plan8.forward(q, k, v, Wq, Wk, g, out8)

        m8 = measure(twin, plan8, step8, args.steps, args.warmup, ws, dev)
        s8 = m8["stage_ms"]
        fp8 = {"workload": twin.name, "dtype": "fp8", "value": aggregate_tflops(m8["flops"], m8["ms_step"], ws),
               "unit": UNIT, "ms_per_step": m8["ms_step"], "steps": args.steps, "warmup": args.warmup,
               "stages": {"kv_pass_ms": s8[0], "query_pass_ms": s8[1], "select_ms": s8[2], "attend_ms": s8[3]},
               "roofline": roofline(twin, s8, m8["flops"]), "clocks": m8["clocks"]}
        plan8.close()
        del out8

    bwd = None
    if not args.no_backward and w.dtype in ("bf16", "f32"):
        # the backward on the same inputs and gain: dout drawn once; a short timed region
        # (each call is long), the same barriers and max over ranks
        dout = synth.make_dout(w, seed=7 + rank, device=dev)
        bwd_warm, bwd_steps = 2, 5

        def bstep():
            plan.backward(q, k, v, Wq, Wk, g, dout)

        mb = measure(w, plan, bstep, bwd_steps, bwd_warm, ws, dev)
        bflops = int(2.5 * mb["flops"])
        bwd = {"ms_per_call": mb["ms_step"], "steps": bwd_steps, "warmup": bwd_warm,
               "value": aggregate_tflops(bflops, mb["ms_step"], ws), "unit": "kept-block TFLOP/s (backward)",
               "flops_per_call": bflops,
               "arithmetic": ("bf16 tensor-core products (tcgen05) with fp32 accumulation; P and dA as bf16 "
                              "hi + lo; the linear branch in fp32" if w.dtype == "bf16" else "fp32"),
               "clocks": mb["clocks"]}
        del dout

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not per_token:
        r = oracle_sample(w, seconds_hint=15.0)
        cpu = {"value": r["value"], "unit": UNIT, "cores": r["cores"], "kind": "oracle",
               "sample": r["sample"], "seconds": r["seconds"]}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if w.dtype != "fp8" else "fp8",
                "data": "synthetic",
                "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "grid": list(w.grid),
                           "d": w.d, "r": w.r, "topk": w.topk, "kept_blocks_per_row": plan.k,
                           "blocks": plan.nb, "kept_block_tflop": flops / 1e12,
                           "gate": {"head": "per-head", "token": "per-token",
                                    "proj": "sigmoid(q . gate_proj + gate_bias)"}[args.gate],
                           "l2": "inputs (3 x 774 MB) larger than L2 (126 MB); no flush",
                           "parallelism": f"replicas x{ws} (independent forward per GPU)"},
                "stages": stages, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "fp8": fp8,
                "backward": bwd,
                "gpu_launches": LAUNCHES_PER_STEP * args.steps, "clocks": clk}
        print(json.dumps(line))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
