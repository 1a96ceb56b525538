"""CPU oracle for the RoLA forward pass — test infrastructure only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may
import this package.  The product library never calls it and shares no code with it.

The arithmetic lives in ``rola_oracle.cpp`` (plain loops; double precision, except the
fp32 block selection).  This
module builds that file with g++ when the shared object is missing or stale, and
marshals numpy arrays in and out.  The definition it follows, and where each step
comes from on the pages about SparkDiffusion / RoLA, is in the header of the C++ file.

Shape conventions: q, k, v are [B, N, H, d]; Wq, Wk are [H, d, r]; g is [H] (a gain per
head), [B, N, H] for a per-token gate (``make_shape(..., gate="token")``), or, for the gate
computed from the query (``gate="proj"``), gate_proj [H, d] followed by gate_bias [H]
(H*(d+1) values), the gain then being sigmoid(q . gate_proj_h + gate_bias_h).
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "rola_oracle.cpp")
_LIB = os.path.join(_HERE, "librola_oracle.so")
_lock = threading.Lock()
_lib = None

BLOCK = 64


def build(force: bool = False) -> str:
    """Compile the oracle (g++ -O3 -fopenmp, no -march, no fast-math)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["g++", "-O3", "-std=c++17", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC])
        os.replace(tmp, _LIB)
    return _LIB


class Shape(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("N", ctypes.c_int),
        ("d", ctypes.c_int), ("r", ctypes.c_int),
        ("grid_t", ctypes.c_int), ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
        ("pairs_t", ctypes.c_int), ("pairs_h", ctypes.c_int), ("pairs_w", ctypes.c_int),
        ("rope_base", ctypes.c_double), ("scale", ctypes.c_double), ("topk", ctypes.c_double),
        ("gate_mode", ctypes.c_int),
    ]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            sp = ctypes.POINTER(Shape)
            lib.rola_oracle_num_blocks.argtypes = [ctypes.c_int]
            lib.rola_oracle_keep_count.argtypes = [ctypes.c_int, ctypes.c_double]
            lib.rola_oracle_positions.argtypes = [sp, P]
            lib.rola_oracle_pool.argtypes = [sp, P, P]
            lib.rola_oracle_select.argtypes = [sp, P, P, P, P, P, P]
            lib.rola_oracle_linear_state.argtypes = [sp, P, P, P, P, P, P]
            lib.rola_oracle_attend_blocks.argtypes = [sp] + [P] * 9 + [ctypes.c_int, P, P, P, P]
            lib.rola_oracle_forward.argtypes = [sp] + [P] * 8
            lib.rola_oracle_threads.restype = ctypes.c_int
            lib.rola_oracle_e4m3_encode.argtypes = [P, P, ctypes.c_size_t]
            lib.rola_oracle_e4m3_decode.argtypes = [P, P, ctypes.c_size_t]
            lib.rola_oracle_quantize_blocks.argtypes = [sp, P, P, P]
            lib.rola_oracle_backward.argtypes = [sp] + [P] * 14
            lib.rola_oracle_backward_sample.argtypes = ([sp] + [P] * 8 + [ctypes.c_int, P, ctypes.c_int, P,
                                                        ctypes.c_int, P] + [P] * 6)
            _lib = lib
    return _lib


def default_pairs(r: int, grid: tuple[int, int, int]) -> tuple[int, int, int]:
    """Rotary pairs per axis (t, h, w) when the caller gives none.

    The pages only say the rotary encoding is 3D.  Reading taken: a 1D grid
    (t = h = 1) puts every pair on the w axis; otherwise h and w get floor(P/3)
    pairs each and t the rest, P = r/2.
    """
    P = r // 2
    if grid[0] == 1 and grid[1] == 1:
        return (0, 0, P)
    hw = P // 3
    return (P - 2 * hw, hw, hw)


GATES = {"head": 0, "token": 1, "proj": 2}


def make_shape(B, H, N, d, r, topk, grid=None, pairs=None, rope_base=10000.0, scale=None,
               gate_per_token=False, gate=None) -> Shape:
    """gate: "head" (g [H]), "token" (g [B, N, H]) or "proj" (g = gate_proj [H, d] then
    gate_bias [H]); ``gate_per_token=True`` is "token"."""
    gate = gate or ("token" if gate_per_token else "head")
    grid = tuple(grid) if grid is not None else (1, 1, N)
    assert grid[0] * grid[1] * grid[2] == N
    pairs = tuple(pairs) if pairs is not None and sum(pairs) > 0 else default_pairs(r, grid)
    assert sum(pairs) == r // 2
    if scale is None or scale == 0:
        scale = 1.0 / math.sqrt(d)
    return Shape(B, H, N, d, r, grid[0], grid[1], grid[2], pairs[0], pairs[1], pairs[2],
                 float(rope_base), float(scale), float(topk), GATES[gate])


def _f32(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float32))


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _gain(s: Shape, g) -> np.ndarray:
    g = _f64(g)
    want = {0: s.H, 1: s.B * s.N * s.H, 2: s.H * (s.d + 1)}[s.gate_mode]
    assert g.size == want, f"g has {g.size} values, the shape needs {want}"
    return g


def _p(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


def num_blocks(N: int) -> int:
    return _load().rola_oracle_num_blocks(N)


def keep_count(nb: int, topk: float) -> int:
    return _load().rola_oracle_keep_count(nb, topk)


def threads() -> int:
    return _load().rola_oracle_threads()


def positions(s: Shape) -> np.ndarray:
    out = np.zeros((s.N, 3), dtype=np.float64)
    _load().rola_oracle_positions(ctypes.byref(s), _p(out))
    return out


def pool(s: Shape, x) -> np.ndarray:
    """fp32 block means [B, H, nb, d] (token-order fp32 sums, one division)."""
    x = _f32(x)
    nb = num_blocks(s.N)
    out = np.zeros((s.B, s.H, nb, s.d), dtype=np.float32)
    _load().rola_oracle_pool(ctypes.byref(s), _p(x), _p(out))
    return out


def select(s: Shape, qbar, kbar):
    """Returns (col_idx [B,H,nb,k] int32, kth, next, amax) — the last three [B,H,nb].

    qbar, kbar are the fp32 block means; scores are fp32 fused multiply-add chains.
    """
    qbar, kbar = _f32(qbar), _f32(kbar)
    nb = num_blocks(s.N)
    k = keep_count(nb, s.topk)
    col = np.zeros((s.B, s.H, nb, k), dtype=np.int32)
    kth = np.zeros((s.B, s.H, nb)); nxt = np.zeros((s.B, s.H, nb)); amax = np.zeros((s.B, s.H, nb))
    _load().rola_oracle_select(ctypes.byref(s), _p(qbar), _p(kbar), _p(col), _p(kth), _p(nxt), _p(amax))
    return col, kth, nxt, amax


def linear_state(s: Shape, k, v, Wk, pos=None):
    """Returns (S [B,H,r,d], z [B,H,r]) in float64."""
    k, v, Wk = _f32(k), _f32(v), _f32(Wk)
    pos = positions(s) if pos is None else _f64(pos)
    S = np.zeros((s.B, s.H, s.r, s.d)); z = np.zeros((s.B, s.H, s.r))
    _load().rola_oracle_linear_state(ctypes.byref(s), _p(k), _p(v), _p(Wk), _p(pos), _p(S), _p(z))
    return S, z


def attend_blocks(s: Shape, q, k, v, Wq, g, col_idx, S, z, blocks, pos=None):
    """Outputs of the listed query blocks.

    blocks: int array [n, 3] of (b, h, i).  Returns (sparse, lin, out), each
    [n, 64, d] float64; rows past N are zero.
    """
    q, k, v, Wq = _f32(q), _f32(k), _f32(v), _f32(Wq)
    g = _gain(s, g); S = _f64(S); z = _f64(z)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    blocks = np.ascontiguousarray(np.asarray(blocks, dtype=np.int32).reshape(-1, 3))
    pos = positions(s) if pos is None else _f64(pos)
    n = blocks.shape[0]
    sp = np.zeros((n, BLOCK, s.d)); li = np.zeros((n, BLOCK, s.d)); out = np.zeros((n, BLOCK, s.d))
    _load().rola_oracle_attend_blocks(ctypes.byref(s), _p(q), _p(k), _p(v), _p(Wq), _p(g), _p(col_idx),
                                      _p(S), _p(z), _p(pos), n, _p(blocks), _p(sp), _p(li), _p(out))
    return sp, li, out


def e4m3_encode(y) -> np.ndarray:
    """e4m3 codes (uint8) of float32 values: nearest, ties to even, saturating at 448."""
    y = _f32(y)
    out = np.zeros(y.shape, dtype=np.uint8)
    _load().rola_oracle_e4m3_encode(_p(y), _p(out), y.size)
    return out


def e4m3_decode(codes) -> np.ndarray:
    """Values (float64) of e4m3 codes; the two NaN codes decode to NaN."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.zeros(codes.shape, dtype=np.float64)
    _load().rola_oracle_e4m3_decode(_p(codes), _p(out), codes.size)
    return out


def quantize_blocks(s: Shape, x):
    """Per-(b, h, 64-token block) e4m3 quantisation of x [B,N,H,d].

    Returns (codes uint8 [B,N,H,d], scales float32 [B,H,nb]); scale = absmax/448 (1 if 0).
    """
    x = _f32(x)
    codes = np.zeros(x.shape, dtype=np.uint8)
    scales = np.zeros((s.B, s.H, num_blocks(s.N)), dtype=np.float32)
    _load().rola_oracle_quantize_blocks(ctypes.byref(s), _p(x), _p(codes), _p(scales))
    return codes, scales


def dequantize_blocks(s: Shape, codes, scales) -> np.ndarray:
    """codes * scale of their (b, h, block), float64 [B,N,H,d]."""
    val = e4m3_decode(codes)
    rep = np.repeat(np.asarray(scales, dtype=np.float64), BLOCK, axis=2)[:, :, :s.N]   # [B,H,N]
    return val * rep.transpose(0, 2, 1)[..., None]


def forward(s: Shape, q, k, v, Wq, Wk, g):
    """Whole forward pass.  Returns (out [B,N,H,d] float64, col_idx [B,H,nb,k])."""
    q, k, v, Wq, Wk = _f32(q), _f32(k), _f32(v), _f32(Wq), _f32(Wk)
    g = _gain(s, g)
    nb = num_blocks(s.N)
    kk = keep_count(nb, s.topk)
    out = np.zeros((s.B, s.N, s.H, s.d))
    col = np.zeros((s.B, s.H, nb, kk), dtype=np.int32)
    _load().rola_oracle_forward(ctypes.byref(s), _p(q), _p(k), _p(v), _p(Wq), _p(Wk), _p(g), _p(out), _p(col))
    return out, col


def backward(s: Shape, q, k, v, Wq, Wk, g, dout, col_idx):
    """Gradients of sum(dout * out) with the kept-block lists col_idx held fixed.

    Returns a dict of float64 arrays: dq, dk, dv [B, N, H, d]; dWq, dWk [H, d, r]; dg
    with the layout of g ([H], [B, N, H], or gate_proj [H, d] then gate_bias [H]).
    """
    q, k, v, Wq, Wk = _f32(q), _f32(k), _f32(v), _f32(Wq), _f32(Wk)
    g = _gain(s, g)
    dout = _f64(dout)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    act = (s.B, s.N, s.H, s.d)
    res = {n: np.zeros(act) for n in ("dq", "dk", "dv")}
    res["dWq"] = np.zeros((s.H, s.d, s.r))
    res["dWk"] = np.zeros((s.H, s.d, s.r))
    res["dg"] = np.zeros(g.size)
    _load().rola_oracle_backward(ctypes.byref(s), _p(q), _p(k), _p(v), _p(Wq), _p(Wk), _p(g), _p(dout),
                                 _p(col_idx), _p(res["dq"]), _p(res["dk"]), _p(res["dv"]), _p(res["dWq"]),
                                 _p(res["dWk"]), _p(res["dg"]))
    return res


def backward_sample(s: Shape, q, k, v, Wq, Wk, g, dout, col_idx, heads, qblocks, kblocks):
    """The backward on a sample (per-head gain only): for the listed heads their dWq, dWk, dg
    (summed over the batch), and for the listed (b, h, i) blocks the 64 rows of dq (qblocks)
    or of dk, dv (kblocks); every listed block's head must be in ``heads``.

    Returns a dict of float64 arrays: dq [nq, 64, d]; dk, dv [nk, 64, d]; dWq, dWk [nh, d, r];
    dg [nh]."""
    assert s.gate_mode == 0
    q, k, v, Wq, Wk = _f32(q), _f32(k), _f32(v), _f32(Wq), _f32(Wk)
    g = _gain(s, g)
    dout = _f64(dout)
    col_idx = np.ascontiguousarray(col_idx, dtype=np.int32)
    heads = np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    qb = np.ascontiguousarray(np.asarray(qblocks, dtype=np.int32).reshape(-1, 3))
    kb = np.ascontiguousarray(np.asarray(kblocks, dtype=np.int32).reshape(-1, 3))
    assert set(qb[:, 1]) | set(kb[:, 1]) <= set(heads.tolist())
    nh, nq, nk = heads.size, qb.shape[0], kb.shape[0]
    res = {"dq": np.zeros((nq, BLOCK, s.d)), "dk": np.zeros((nk, BLOCK, s.d)), "dv": np.zeros((nk, BLOCK, s.d)),
           "dWq": np.zeros((nh, s.d, s.r)), "dWk": np.zeros((nh, s.d, s.r)), "dg": np.zeros(nh)}
    _load().rola_oracle_backward_sample(ctypes.byref(s), _p(q), _p(k), _p(v), _p(Wq), _p(Wk), _p(g), _p(dout),
                                        _p(col_idx), nh, _p(heads), nq, _p(qb), nk, _p(kb), _p(res["dq"]),
                                        _p(res["dk"]), _p(res["dv"]), _p(res["dWq"]), _p(res["dWk"]), _p(res["dg"]))
    return res
