"""Shared helpers of the parity tests: run the CUDA library through its C ABI and the
CPU oracle on the same seeded inputs, and compare them.

Tolerances (stated by the operator's specification, tied to the input type):
  * block lists: bit-exact (the selection is defined in fp32 with a stated order);
  * pooled means: bit-exact;
  * fp32 configuration: max |out - oracle| <= 1e-4;
  * bf16 configuration: |out - oracle| <= 2e-2 * RMS(oracle out) + half a bf16 ulp;
  * fp8 configuration:  RMS(out - oracle) <= 6e-2 * RMS(oracle out), over the compared
    elements (a normwise bound: an elementwise one is out of reach of e4m3 V, whose 3
    mantissa bits alone move an output dominated by one value by up to 2^-4 of it), plus
    a guard on every 64-token query block: RMS of its error <= 0.08 * RMS(oracle out)
    (a CPU emulation of the exact quantisation gives at most 0.047 per block on these
    inputs; the GPU cases measured up to 0.060 on the smallest ragged problems, where a
    block's few valid rows weigh most).
The oracle's double-precision output (before its own final rounding) is the reference.
The operator's last step rounds out once to bf16; that rounding alone moves an element
by up to half a bf16 ulp (2^-8 of its magnitude), which on these outputs (max/RMS of
6-15) exceeds 2e-2 * RMS by itself.  The RMS-relative tolerance therefore bounds the
computation error, and each element is also allowed the half ulp its own rounding costs.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola

TOL_REL = {"bf16": 2e-2, "fp8": 6e-2}
FP8_BLOCK_GUARD = 0.08
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


def half_ulp_bf16(x: np.ndarray) -> np.ndarray:
    """Half the spacing of bf16 numbers at |x| (8 significant bits)."""
    a = np.maximum(np.abs(x), np.finfo(np.float32).tiny)
    e = np.floor(np.log2(a))
    return np.ldexp(1.0, (e - 8).astype(np.int64))


def check_out(got: np.ndarray, want: np.ndarray, dtype: str, what=""):
    err = np.abs(got - want)
    if dtype == "f32":
        assert err.max() <= TOL_ABS_F32, f"{what}: max abs err {err.max():.3e} > {TOL_ABS_F32}"
        return err.max(), None
    rms = math.sqrt(float(np.mean(want ** 2)))
    allow = TOL_REL[dtype] * rms + half_ulp_bf16(np.maximum(np.abs(want), np.abs(got)))
    excess = err - allow
    worst = int(np.argmax(excess))
    compute_err = float(np.max(err - half_ulp_bf16(np.maximum(np.abs(want), np.abs(got)))))
    assert excess.flat[worst] <= 0, (
        f"{what}: |out - oracle| = {err.flat[worst]:.3e} at {want.flat[worst]:.4f} exceeds "
        f"{TOL_REL[dtype]} * rms {rms:.3e} + half ulp; computation error bound {compute_err:.3e}")
    return err.max(), rms


def check_out_fp8(got: np.ndarray, want: np.ndarray, valid: np.ndarray, what="", tol=None):
    """Normwise fp8 check on [n, 64, d] query blocks (rows past N masked by `valid`).
    Returns (normwise error / RMS, worst block's error RMS / RMS)."""
    tol = TOL_REL["fp8"] if tol is None else tol
    m = valid[..., None].astype(np.float64)
    cnt = m.sum() * got.shape[-1]
    rms = math.sqrt(float(np.sum((want * m) ** 2) / cnt))
    err2 = ((got - want) * m) ** 2
    norm = math.sqrt(float(err2.sum() / cnt)) / rms
    per_block = np.sqrt(err2.sum(axis=(1, 2)) / np.maximum(m.sum(axis=(1, 2)) * got.shape[-1], 1)) / rms
    worst = float(per_block.max())
    assert norm <= tol, f"{what}: normwise error {norm:.3e} of RMS exceeds {tol}"
    assert worst <= FP8_BLOCK_GUARD, f"{what}: a query block's error RMS is {worst:.3e} of RMS"
    return norm, worst
