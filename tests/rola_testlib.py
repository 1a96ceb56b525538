"""Shared helpers of the parity tests: run the CUDA library through its C ABI and the
CPU oracle on the same seeded inputs, and compare them.

Tolerances (stated by the operator's specification, tied to the input type):
  * block lists: bit-exact (the selection is defined in fp32 with a stated order);
  * pooled means: bit-exact;
  * fp32 configuration: max |out - oracle| <= 1e-4;
  * bf16 configuration: max |out - oracle| <= 2e-2 * RMS(oracle out);
  * fp8 configuration:  max |out - oracle| <= 6e-2 * RMS(oracle out).
The oracle's double-precision output (before its own final rounding) is the reference.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola

TOL_REL = {"bf16": 2e-2, "fp8": 6e-2}
TOL_ABS_F32 = 1e-4


def shape_of(w) -> O.Shape:
    return O.make_shape(w.B, w.H, w.N, w.d, w.r, w.topk, grid=w.grid, pairs=w.pairs)


def np32(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy()


def run_gpu(w, inp, plan=None):
    """Runs the three steps through the C ABI; returns a dict of host results."""
    plan = plan or rola.Plan.for_workload(w)
    out = torch.empty_like(inp["q"])
    plan.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], out)
    col = plan.block_lists()
    qbar, kbar = plan.pooled()
    S, z = plan.state()
    status = plan.poll_status()
    return {"plan": plan, "out": out, "col": col.cpu().numpy(), "qbar": qbar.cpu().numpy(),
            "kbar": kbar.cpu().numpy(), "S": S.cpu().numpy(), "z": z.cpu().numpy(),
            "status": status}


def host_inputs(inp):
    return {k: np32(v) for k, v in inp.items()}


def sample_blocks(w, n_heads=4, n_blocks=16, seed=0):
    """Seeded (b, h, i) sample that always includes the first and the last (tail) block."""
    rng = np.random.default_rng(seed)
    heads = sorted(set(rng.choice(w.H, size=min(n_heads, w.H), replace=False).tolist()))
    out = []
    for b in range(w.B):
        for h in heads:
            idx = set(rng.choice(w.nb, size=min(n_blocks, w.nb), replace=False).tolist())
            idx |= {0, w.nb - 1}
            out += [(b, h, i) for i in sorted(idx)]
    return np.array(out, dtype=np.int32)


def gather_blocks(out_gpu: np.ndarray, blocks, N) -> tuple[np.ndarray, np.ndarray]:
    """GPU rows of the listed query blocks as [n, 64, d] plus a validity mask."""
    B, _, H, d = out_gpu.shape
    res = np.zeros((len(blocks), 64, d), dtype=np.float64)
    valid = np.zeros((len(blocks), 64), dtype=bool)
    for t, (b, h, i) in enumerate(blocks):
        n1 = min(N, 64 * i + 64)
        res[t, :n1 - 64 * i] = out_gpu[b, 64 * i:n1, h]
        valid[t, :n1 - 64 * i] = True
    return res, valid


def check_out(got: np.ndarray, want: np.ndarray, dtype: str, what=""):
    err = np.abs(got - want).max()
    if dtype == "f32":
        assert err <= TOL_ABS_F32, f"{what}: max abs err {err:.3e} > {TOL_ABS_F32}"
        return err, None
    rms = math.sqrt(float(np.mean(want ** 2)))
    assert err <= TOL_REL[dtype] * rms, f"{what}: max abs err {err:.3e} > {TOL_REL[dtype]} * rms {rms:.3e}"
    return err, rms
