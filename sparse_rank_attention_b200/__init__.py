"""RoLA attention forward on NVIDIA B200 (sm_100a): thin Python binding of librola.so.

RoLA ("Rotary-Positioned Low-Rank Linear Attention", the sparse attention module of
SparkDiffusion) adds a rank-r linear-attention branch with 3D rotary positions to a
block-sparse softmax branch that keeps the top-k fraction of 64-token key blocks per
query block.  The operator, its layouts and error rules are documented in
``include/rola.h``; every step runs in the library's CUDA kernels.  This module only
marshals torch tensors (device memory, the current stream) into the C ABI.

Layouts: q, k, v, out [B, N, H, d]; Wq, Wk [H, d, r]; g [H] fp32 — contiguous, on the
same CUDA device.  fp32 tensors select the fp32 configuration, bf16 tensors the bf16 one;
``dtype="fp8"`` takes bf16 tensors and quantises inside.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librola.so")

ROLA_F32, ROLA_BF16, ROLA_FP8_E4M3 = 0, 1, 2
DTYPES = {"f32": ROLA_F32, "bf16": ROLA_BF16, "fp8": ROLA_FP8_E4M3}
ROLA_DEBUG_STALL_WAIT = 1
# how the gain of the linear branch is given (rola_gate): g [H], g [B, N, H], or the gate
# computed from the query, g = gate_proj [H, d] followed by gate_bias [H]
GATES = {"head": 0, "token": 1, "proj": 2}

STATUS = {0: "ROLA_OK", 1: "ROLA_ERR_INVALID_ARG", 2: "ROLA_ERR_UNSUPPORTED",
          3: "ROLA_ERR_WORKSPACE", 4: "ROLA_ERR_CUDA", 5: "ROLA_ERR_DEVICE_TIMEOUT",
          6: "ROLA_ERR_DEVICE_BOUNDS", 7: "ROLA_ERR_RANGE"}

EXPORTS = ("rola_params_default", "rola_keep_count", "rola_workspace_size", "rola_plan",
           "rola_plan_destroy", "rola_select_blocks", "rola_linear_state", "rola_attend",
           "rola_forward", "rola_get_block_lists", "rola_get_pooled", "rola_get_linear_state",
           "rola_poll_device_status", "rola_set_debug", "rola_status_string",
           "rola_select_blocks_noalloc", "rola_get_fp8_copies", "rola_profile_stages",
           "rola_get_stage_times", "rola_get_attend_redo_count", "rola_eval_exp2",
           "rola_backward_workspace_size", "rola_backward", "rola_get_block_scores")


class RolaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({_lib_status_string(code)})")


class RolaParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
        ("d", ctypes.c_int), ("r", ctypes.c_int), ("block", ctypes.c_int),
        ("topk", ctypes.c_double),
        ("grid_t", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("rope_pairs_t", ctypes.c_int), ("rope_pairs_h", ctypes.c_int),
        ("rope_pairs_w", ctypes.c_int),
        ("rope_base", ctypes.c_double), ("softmax_scale", ctypes.c_float),
        ("dtype", ctypes.c_int), ("gate", ctypes.c_int),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """Load librola.so; raises if it has not been built (no fallback path exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m sparse_rank_attention_b200.build` "
            "(or __graft_entry__.build()). There is no CPU or PyTorch fallback.")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    pp = ctypes.POINTER(RolaParams)
    i32 = ctypes.c_int
    for name, args in {
        "rola_params_default": [pp],
        "rola_keep_count": [pp, ctypes.POINTER(i32), ctypes.POINTER(i32)],
        "rola_workspace_size": [pp, ctypes.POINTER(ctypes.c_size_t)],
        "rola_plan": [pp, P, ctypes.c_size_t, ctypes.POINTER(P)],
        "rola_select_blocks": [P, P, P, P],
        "rola_linear_state": [P, P, P, P, P],
        "rola_attend": [P, P, P, P, P, P, P, P],
        "rola_forward": [P, P, P, P, P, P, P, P, P],
        "rola_get_block_lists": [P, P, P],
        "rola_get_pooled": [P, P, P, P],
        "rola_get_block_scores": [P, P, P, P],
        "rola_get_linear_state": [P, P, P, P],
        "rola_poll_device_status": [P, P],
        "rola_set_debug": [P, i32, i32],
        "rola_select_blocks_noalloc": [pp, P, P, P, P],
        "rola_get_fp8_copies": [P, P, P, P, P, P, P, P],
        "rola_profile_stages": [P, i32],
        "rola_get_attend_redo_count": [P, ctypes.POINTER(i32), P],
        "rola_eval_exp2": [P, P, ctypes.c_int64, i32, P],
        "rola_backward_workspace_size": [pp, ctypes.POINTER(ctypes.c_size_t)],
        "rola_backward": [P] * 15 + [ctypes.c_size_t, P],
        "rola_get_stage_times": [P, ctypes.POINTER(ctypes.c_float), i32, ctypes.POINTER(i32),
                                 ctypes.POINTER(i32)],
    }.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = i32
    lib.rola_plan_destroy.argtypes = [P]
    lib.rola_plan_destroy.restype = None
    lib.rola_status_string.argtypes = [i32]
    lib.rola_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def eval_exp2(x, mode: int):
    """2^x of a contiguous fp32 CUDA tensor through rola_eval_exp2 (mode 0: ex2.approx, 1: the
    polynomial on the FMA pipe), the device functions of the attention kernels' softmax."""
    assert x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()
    y = torch.empty_like(x)
    _check(load().rola_eval_exp2(x.data_ptr(), y.data_ptr(), x.numel(), mode,
                                 torch.cuda.current_stream().cuda_stream), "rola_eval_exp2")
    return y


def _lib_status_string(code: int) -> str:
    try:
        return load().rola_status_string(code).decode()
    except Exception:  # noqa: BLE001 - message only
        return "?"


def _check(code: int, where: str):
    if code != 0:
        raise RolaError(code, where)


def _gate(gate, gate_per_token) -> int:
    if gate is None:
        gate = "token" if gate_per_token else "head"
    return GATES[gate] if isinstance(gate, str) else int(gate)


def make_params(B, H, N, d, r, topk, grid=None, pairs=(0, 0, 0), rope_base=10000.0,
                softmax_scale=0.0, dtype="bf16", gate_per_token=False, gate=None) -> RolaParams:
    """rola_params; gate is "head", "token" or "proj" (``gate_per_token=True`` = "token")."""
    p = RolaParams()
    load().rola_params_default(ctypes.byref(p))
    grid = tuple(grid) if grid is not None else (1, 1, N)
    p.B, p.H, p.N, p.d, p.r = B, H, N, d, r
    p.topk = float(topk)
    p.grid_t, p.grid_h, p.grid_w = grid
    p.rope_pairs_t, p.rope_pairs_h, p.rope_pairs_w = pairs
    p.rope_base = float(rope_base)
    p.softmax_scale = float(softmax_scale)
    p.dtype = DTYPES[dtype] if isinstance(dtype, str) else int(dtype)
    p.gate = _gate(gate, gate_per_token)
    return p


def keep_count(params: RolaParams) -> tuple[int, int]:
    nb, k = ctypes.c_int(), ctypes.c_int()
    _check(load().rola_keep_count(ctypes.byref(params), ctypes.byref(nb), ctypes.byref(k)),
           "rola_keep_count")
    return nb.value, k.value


def workspace_size(params: RolaParams) -> int:
    n = ctypes.c_size_t()
    _check(load().rola_workspace_size(ctypes.byref(params), ctypes.byref(n)), "rola_workspace_size")
    return n.value


def _ptr(t: torch.Tensor | None):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


class Plan:
    """A rola_plan bound to a workspace tensor allocated here with torch."""

    def __init__(self, B, H, N, d, r, topk, grid=None, pairs=(0, 0, 0), rope_base=10000.0,
                 softmax_scale=0.0, dtype="bf16", device="cuda", gate_per_token=False, gate=None):
        self.params = make_params(B, H, N, d, r, topk, grid, pairs, rope_base, softmax_scale, dtype,
                                  gate_per_token, gate)
        self.dtype = dtype
        self.nb, self.k = keep_count(self.params)
        self.workspace_bytes = workspace_size(self.params)
        self.workspace = torch.empty(self.workspace_bytes, dtype=torch.uint8, device=device)
        h = ctypes.c_void_p()
        _check(load().rola_plan(ctypes.byref(self.params), _ptr(self.workspace),
                                self.workspace_bytes, ctypes.byref(h)), "rola_plan")
        self._h = h

    @classmethod
    def for_workload(cls, w, device="cuda", gate_per_token=False, gate=None):
        return cls(w.B, w.H, w.N, w.d, w.r, w.topk, w.grid, w.pairs, dtype=w.dtype, device=device,
                   gate_per_token=gate_per_token, gate=gate)

    def close(self):
        if getattr(self, "_h", None):
            load().rola_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # noqa: BLE001 - interpreter shutdown
            pass

    # ---- steps
    def select_blocks(self, q, k, stream=None):
        _check(load().rola_select_blocks(self._h, _ptr(q), _ptr(k), _stream(stream)),
               "rola_select_blocks")

    def linear_state(self, k, v, Wk, stream=None):
        _check(load().rola_linear_state(self._h, _ptr(k), _ptr(v), _ptr(Wk), _stream(stream)),
               "rola_linear_state")

    def attend(self, q, k, v, Wq, g, out, stream=None):
        _check(load().rola_attend(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(Wq), _ptr(g),
                                  _ptr(out), _stream(stream)), "rola_attend")
        return out

    def forward(self, q, k, v, Wq, Wk, g, out=None, stream=None):
        if out is None:
            out = torch.empty_like(q)
        _check(load().rola_forward(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(Wq), _ptr(Wk),
                                   _ptr(g), _ptr(out), _stream(stream)), "rola_forward")
        return out

    def backward(self, q, k, v, Wq, Wk, g, dout, stream=None):
        """Gradients of sum(dout * out) through rola_backward (kept-block lists fixed).

        Returns a dict of fp32 tensors: dq, dk, dv [B, N, H, d]; dWq, dWk [H, d, r]; dg with
        the layout of g.  The backward scratch is allocated once per plan and kept."""
        p = self.params
        dev = self.workspace.device
        if getattr(self, "bwd_workspace", None) is None:
            n = ctypes.c_size_t()
            _check(load().rola_backward_workspace_size(ctypes.byref(p), ctypes.byref(n)),
                   "rola_backward_workspace_size")
            self.bwd_workspace = torch.empty(n.value, dtype=torch.uint8, device=dev)
        act = (p.B, p.N, p.H, p.d)
        res = {n: torch.empty(act, dtype=torch.float32, device=dev) for n in ("dq", "dk", "dv")}
        res["dWq"] = torch.empty((p.H, p.d, p.r), dtype=torch.float32, device=dev)
        res["dWk"] = torch.empty((p.H, p.d, p.r), dtype=torch.float32, device=dev)
        res["dg"] = torch.empty(g.numel(), dtype=torch.float32, device=dev)
        _check(load().rola_backward(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(Wq), _ptr(Wk), _ptr(g),
                                    _ptr(dout), *[_ptr(res[n]) for n in ("dq", "dk", "dv", "dWq", "dWk", "dg")],
                                    _ptr(self.bwd_workspace), self.bwd_workspace.numel(), _stream(stream)),
               "rola_backward")
        return res

    # ---- inspection
    def block_lists(self, stream=None) -> torch.Tensor:
        p = self.params
        t = torch.empty((p.B, p.H, self.nb, self.k), dtype=torch.int32, device=self.workspace.device)
        _check(load().rola_get_block_lists(self._h, _ptr(t), _stream(stream)), "rola_get_block_lists")
        return t

    def pooled(self, stream=None):
        p = self.params
        qb = torch.empty((p.B, p.H, self.nb, p.d), dtype=torch.float32, device=self.workspace.device)
        kb = torch.empty_like(qb)
        _check(load().rola_get_pooled(self._h, _ptr(qb), _ptr(kb), _stream(stream)), "rola_get_pooled")
        return qb, kb

    def block_scores(self, stream=None):
        """The tensor-core block scores [B, H, nb, nb] of the last selection and the key-block
        norms [B, H, nb] that bound their error."""
        p = self.params
        sc = torch.empty((p.B, p.H, self.nb, self.nb), dtype=torch.float32, device=self.workspace.device)
        kn = torch.empty((p.B, p.H, self.nb), dtype=torch.float32, device=self.workspace.device)
        _check(load().rola_get_block_scores(self._h, _ptr(sc), _ptr(kn), _stream(stream)), "rola_get_block_scores")
        return sc, kn

    def state(self, stream=None):
        p = self.params
        S = torch.empty((p.B, p.H, p.r, p.d), dtype=torch.float32, device=self.workspace.device)
        z = torch.empty((p.B, p.H, p.r), dtype=torch.float32, device=self.workspace.device)
        _check(load().rola_get_linear_state(self._h, _ptr(S), _ptr(z), _stream(stream)),
               "rola_get_linear_state")
        return S, z

    def fp8_copies(self, stream=None):
        """(q8, k8, v8) uint8 [B,N,H,d] e4m3 codes and (sq, sk, sv) fp32 [B,H,nb] scales."""
        p = self.params
        dev = self.workspace.device
        codes = [torch.empty((p.B, p.N, p.H, p.d), dtype=torch.uint8, device=dev) for _ in range(3)]
        scales = [torch.empty((p.B, p.H, self.nb), dtype=torch.float32, device=dev) for _ in range(3)]
        _check(load().rola_get_fp8_copies(self._h, *[_ptr(t) for t in codes + scales], _stream(stream)),
               "rola_get_fp8_copies")
        return codes, scales

    def profile_stages(self, enable: bool = True):
        """Record CUDA events between the stages of later forward calls (see rola.h)."""
        _check(load().rola_profile_stages(self._h, int(bool(enable))), "rola_profile_stages")

    def stage_times(self) -> tuple[list[float], int]:
        """(summed milliseconds per stage, number of recorded forward calls); clears the record."""
        ms = (ctypes.c_float * 8)()
        ns, nc = ctypes.c_int(), ctypes.c_int()
        _check(load().rola_get_stage_times(self._h, ms, 8, ctypes.byref(ns), ctypes.byref(nc)),
               "rola_get_stage_times")
        return [ms[i] for i in range(ns.value)], nc.value

    def attend_redo_count(self, stream=None) -> int:
        """Tiles the last attention call recomputed in its careful pass (synchronises)."""
        n = ctypes.c_int()
        _check(load().rola_get_attend_redo_count(self._h, ctypes.byref(n), _stream(stream)),
               "rola_get_attend_redo_count")
        return n.value

    def poll_status(self, stream=None) -> int:
        """Synchronises the stream; returns the device status code (0 = ok), clearing it."""
        return load().rola_poll_device_status(self._h, _stream(stream))

    def set_debug(self, flags: int, limit_us: int = 0):
        _check(load().rola_set_debug(self._h, flags, limit_us), "rola_set_debug")


def select_blocks_noalloc(params: RolaParams, q, k, col_idx, stream=None) -> int:
    """Block selection into the caller's col_idx [B,H,nb,k] int32 with no device allocation
    (the library's own fixed scratch); returns the rola_status code."""
    return load().rola_select_blocks_noalloc(ctypes.byref(params), _ptr(q), _ptr(k), _ptr(col_idx),
                                             _stream(stream))


def forward(q, k, v, Wq, Wk, g, topk, grid=None, pairs=(0, 0, 0), rope_base=10000.0,
            softmax_scale=0.0, dtype=None, out=None, gate=None):
    """One-shot RoLA forward (builds a plan and workspace for this call).  g is [H], or
    [B, N, H] for a per-token gate, or gate_proj [H, d] then gate_bias [H] with
    ``gate="proj"``."""
    B, N, H, d = q.shape
    r = Wq.shape[-1]
    if dtype is None:
        dtype = "f32" if q.dtype == torch.float32 else "bf16"
    plan = Plan(B, H, N, d, r, topk, grid, pairs, rope_base, softmax_scale, dtype, q.device,
                gate_per_token=g.dim() > 1, gate=gate)
    try:
        return plan.forward(q, k, v, Wq, Wk, g, out)
    finally:
        torch.cuda.current_stream().synchronize()
        plan.close()


__all__ = ["Plan", "forward", "select_blocks_noalloc", "load", "make_params", "keep_count", "workspace_size", "RolaError",
           "RolaParams", "EXPORTS", "LIB_PATH", "ROLA_DEBUG_STALL_WAIT", "GATES"]
