"""Seeded synthetic inputs for RoLA forward workloads.

This module is shared by the tests, the benchmark and the smoke check, for both the
CUDA library and the CPU oracle.  It holds no step of the method: it only draws the
tensors (q, k, v, Wq, Wk, g) with the shapes and value distributions of the
Wan2.1-shaped workloads, from a seeded ``torch.Generator`` on the requested device.
Values depend on the device the generator runs on; every comparison draws once and
hands the same tensors to both sides.

Distributions (the pages only name the video models, so these stand in for real
activations; no model weights or data are involved):
  * ``block_offset``: q, k, v = N(0, 1) plus one N(0, 0.5^2) vector per (head, 64-token
    block) shared by the tokens of that block, drawn independently per tensor, so that
    block energies differ.
  * ``sin_field``: q, k, v = N(0, 1) plus 0.5 * sin(w_t*t + w_y*y + w_x*x + phase), one
    (w_t, w_y, w_x) ~ U(0, pi/8) and phase ~ U(0, 2*pi) per (head, channel), drawn
    independently per tensor: a smooth 3D field over the (t, y, x) latent grid.
  * Wq, Wk ~ N(0, 1/d) of shape [H, d, r]; g ~ U(0.1, 1) per head unless fixed.
Inputs are rounded to the workload's input dtype (bf16 for the bf16 and fp8 runs).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch

BLOCK = 64


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    r: int
    topk: float
    grid: tuple          # (t, h, w) latent grid, product == N
    dtype: str           # "f32" | "bf16" | "fp8"
    dist: str            # "block_offset" | "sin_field"
    g_const: float | None = None   # fixed gain for every head, else U(0.1, 1)
    pairs: tuple = (0, 0, 0)       # rotary pairs per axis; zeros = library default

    @property
    def nb(self) -> int:
        return (self.N + BLOCK - 1) // BLOCK


WORKLOADS = {
    # Tiny fp32 correctness case: 16x16 block grid, 4 kept key blocks per query block.
    "tiny_f32_h2_n1024": Workload("tiny_f32_h2_n1024", 1, 2, 1024, 64, 16, 0.25, (1, 1, 1024),
                                  "f32", "block_offset", g_const=0.5),
    # Wan2.1-T2V-1.3B at 480P: 21x30x52 latent grid, 12 heads, 90 % sparsity.
    "wan21_1p3b_480p": Workload("wan21_1p3b_480p", 1, 12, 32760, 128, 32, 0.10, (21, 30, 52),
                                "bf16", "sin_field"),
    # Wan2.1-T2V-14B at 480P: 40 heads, 95 % sparsity.
    "wan21_14b_480p": Workload("wan21_14b_480p", 1, 40, 32760, 128, 32, 0.05, (21, 30, 52),
                               "bf16", "sin_field"),
    # Wan2.1-T2V-14B at 720P: 21x45x80 grid, 40 heads, 97 % sparsity (bf16 and fp8).
    "wan21_14b_720p": Workload("wan21_14b_720p", 1, 40, 75600, 128, 32, 0.03, (21, 45, 80),
                               "bf16", "sin_field"),
    "wan21_14b_720p_fp8": Workload("wan21_14b_720p_fp8", 1, 40, 75600, 128, 32, 0.03,
                                   (21, 45, 80), "fp8", "sin_field"),
}
# Sparsity sweep at the 14B-480P shape; topk = 1.0 with g = 0 is plain dense attention.
for _t in (0.03, 0.05, 0.10, 0.25, 1.0):
    _n = f"wan21_14b_480p_topk{_t:g}"
    WORKLOADS[_n] = replace(WORKLOADS["wan21_14b_480p"], name=_n, topk=_t)
WORKLOADS["wan21_14b_480p_fp8"] = replace(WORKLOADS["wan21_14b_480p"], name="wan21_14b_480p_fp8",
                                          dtype="fp8")
# Classifier-free guidance batch of the multi-step CFG sampler (the pages' teacher and
# reference runs): the conditional and unconditional inputs as B = 2, 14B at 480P.
WORKLOADS["wan21_14b_480p_cfg_b2"] = replace(WORKLOADS["wan21_14b_480p"], name="wan21_14b_480p_cfg_b2",
                                             B=2)
WORKLOADS["wan21_14b_480p_dense_g0"] = replace(WORKLOADS["wan21_14b_480p"],
                                               name="wan21_14b_480p_dense_g0", topk=1.0,
                                               g_const=0.0)
# Image-to-video at 480P (the pages' I2V example keeps 0.05): the latent grid follows the
# input image's aspect ratio and the frame count (NUM_FRAMES, ASPECT_RATIO,
# FIXED_RESOLUTION), so the sequence length and the 3D grid change with them.
#   portrait 480x832: 21 x 52 x 30 (same N as landscape, transposed grid);
#   square 624x624:   21 x 39 x 39 = 31941 tokens (a 5-token last block);
#   49 frames:        13 x 30 x 52 = 20280 tokens.
WORKLOADS["wan21_14b_i2v_480p_portrait"] = replace(WORKLOADS["wan21_14b_480p"], name="wan21_14b_i2v_480p_portrait",
                                                   grid=(21, 52, 30))
WORKLOADS["wan21_14b_i2v_480p_square"] = replace(WORKLOADS["wan21_14b_480p"], name="wan21_14b_i2v_480p_square",
                                                 N=31941, grid=(21, 39, 39))
WORKLOADS["wan21_14b_i2v_480p_49f"] = replace(WORKLOADS["wan21_14b_480p"], name="wan21_14b_i2v_480p_49f",
                                              N=20280, grid=(13, 30, 52))
# Wan2.2-A14B (two experts of the 14B attention shape, high- and low-noise) with the keep
# ratio of the pages' Wan 2.2 example, 0.1, at 480P and 720P.
WORKLOADS["wan22_a14b_480p"] = replace(WORKLOADS["wan21_14b_480p"], name="wan22_a14b_480p", topk=0.10)
WORKLOADS["wan22_a14b_720p"] = replace(WORKLOADS["wan21_14b_720p"], name="wan22_a14b_720p", topk=0.10)


def custom(name="custom", B=1, H=2, N=1024, d=64, r=16, topk=0.25, grid=None, dtype="bf16",
           dist="sin_field", g_const=None, pairs=(0, 0, 0)) -> Workload:
    grid = tuple(grid) if grid is not None else (1, 1, N)
    return Workload(name, B, H, N, d, r, topk, grid, dtype, dist, g_const, tuple(pairs))


def _torch_dtype(w: Workload):
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _grid_coords(w: Workload, n0: int, n1: int, device):
    n = torch.arange(n0, n1, device=device, dtype=torch.int64)
    gt, gh, gw = w.grid
    x = (n % gw).to(torch.float32)
    y = ((n // gw) % gh).to(torch.float32)
    t = (n // (gw * gh)).to(torch.float32)
    return t, y, x


def _activation(w: Workload, gen: torch.Generator, device, chunk: int = 8192) -> torch.Tensor:
    out = torch.empty((w.B, w.N, w.H, w.d), dtype=_torch_dtype(w), device=device)
    if w.dist == "block_offset":
        off = torch.randn((w.B, w.nb, w.H, w.d), generator=gen, device=device) * 0.5
        for n0 in range(0, w.N, chunk):
            n1 = min(w.N, n0 + chunk)
            x = torch.randn((w.B, n1 - n0, w.H, w.d), generator=gen, device=device)
            blk = torch.arange(n0, n1, device=device) // BLOCK
            x += off[:, blk]
            out[:, n0:n1] = x.to(out.dtype)
    elif w.dist == "sin_field":
        omega = torch.rand((3, w.H, w.d), generator=gen, device=device) * (math.pi / 8)
        phase = torch.rand((w.H, w.d), generator=gen, device=device) * (2 * math.pi)
        for n0 in range(0, w.N, chunk):
            n1 = min(w.N, n0 + chunk)
            t, y, x_ = _grid_coords(w, n0, n1, device)
            ang = (t[:, None, None] * omega[0] + y[:, None, None] * omega[1]
                   + x_[:, None, None] * omega[2] + phase)
            x = torch.randn((w.B, n1 - n0, w.H, w.d), generator=gen, device=device)
            x += 0.5 * torch.sin(ang)[None]
            out[:, n0:n1] = x.to(out.dtype)
    else:
        raise ValueError(f"unknown distribution {w.dist}")
    return out


def make_inputs(w: Workload, seed: int = 0, device="cpu") -> dict:
    """Draw q, k, v [B,N,H,d], Wq, Wk [H,d,r] and g [H] (fp32) for workload ``w``."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q = _activation(w, gen, device)
    k = _activation(w, gen, device)
    v = _activation(w, gen, device)
    std = 1.0 / math.sqrt(w.d)
    Wq = (torch.randn((w.H, w.d, w.r), generator=gen, device=device) * std).to(_torch_dtype(w))
    Wk = (torch.randn((w.H, w.d, w.r), generator=gen, device=device) * std).to(_torch_dtype(w))
    if w.g_const is not None:
        g = torch.full((w.H,), float(w.g_const), dtype=torch.float32, device=device)
    else:
        g = (torch.rand((w.H,), generator=gen, device=device) * 0.9 + 0.1).to(torch.float32)
    return {"q": q, "k": k, "v": v, "Wq": Wq, "Wk": Wk, "g": g}


def make_gate(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """A per-token, per-head gate [B, N, H] (fp32, uniform in (0, 1), the range of a
    sigmoid gate) for workload ``w``, from its own seeded stream."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.rand((w.B, w.N, w.H), generator=gen, device=device, dtype=torch.float32)


def make_gate_proj(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """Parameters of a gate computed from the query (the gate_proj / gate_bias pair): one
    fp32 buffer of H*(d+1) values, gate_proj [H, d] ~ N(0, 1/d) followed by gate_bias [H]
    ~ U(-0.5, 0.5), from its own seeded stream."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    wg = torch.randn((w.H, w.d), generator=gen, device=device, dtype=torch.float32) / math.sqrt(w.d)
    bg = torch.rand((w.H,), generator=gen, device=device, dtype=torch.float32) - 0.5
    return torch.cat([wg.reshape(-1), bg]).contiguous()


def make_dout(w: Workload, seed: int = 0, device="cpu") -> torch.Tensor:
    """An upstream gradient dout [B, N, H, d] ~ N(0, 1) in the workload's input dtype (bf16,
    or fp32), from its own seeded stream: the cotangent a backward call consumes."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return torch.randn((w.B, w.N, w.H, w.d), generator=gen, device=device).to(_torch_dtype(w))


__all__ = ["Workload", "WORKLOADS", "BLOCK", "custom", "make_inputs", "make_gate", "make_gate_proj",
           "make_dout"]
