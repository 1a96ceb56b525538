"""C-ABI checks that need no GPU: the library loads, exports every declared entry
point, and its host-side logic (parameter checks, keep count, workspace sizing,
plan creation) behaves as include/rola.h states."""
import ctypes
import os
import re

import pytest

import sparse_rank_attention_b200 as rola
from sparse_rank_attention_b200 import build as rbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def _built():
    rbuild.build()


def _declared():
    text = open(os.path.join(ROOT, "include", "rola.h")).read()
    return sorted(set(re.findall(r"ROLA_API\s+[\w\s\*]+?\b(rola_\w+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    names = _declared()
    assert len(names) >= 15
    lib = rola.load()
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(rola.EXPORTS)


def _params(**kw):
    base = dict(B=1, H=2, N=1000, d=64, r=16, topk=0.25)
    base.update(kw)
    return rola.make_params(**base)


def test_keep_count_and_blocks():
    assert rola.keep_count(_params(N=32760, topk=0.10, d=128, r=32)) == (512, 52)
    assert rola.keep_count(_params(N=75600, topk=0.03, d=128, r=32)) == (1182, 36)
    assert rola.keep_count(_params(N=32760, topk=0.05)) == (512, 26)
    assert rola.keep_count(_params(N=6400, topk=0.07)) == (100, 7)
    assert rola.keep_count(_params(N=64, topk=0.01)) == (1, 1)
    assert rola.keep_count(_params(N=1000, topk=1.0)) == (16, 16)


@pytest.mark.parametrize("kw,code", [
    (dict(d=96), 2), (dict(r=8), 2), (dict(N=0), 1), (dict(topk=0.0), 1), (dict(topk=1.5), 1),
    (dict(grid=(2, 2, 7)), 1), (dict(pairs=(1, 1, 1)), 1), (dict(pairs=(-1, 5, 4)), 1),
    (dict(rope_base=1.0), 1), (dict(softmax_scale=-1.0), 1), (dict(dtype=7), 1),
    (dict(N=64 * 7000), 2),
])
def test_invalid_params_rejected(kw, code):
    p = _params(**kw)
    n = ctypes.c_size_t()
    assert rola.load().rola_workspace_size(ctypes.byref(p), ctypes.byref(n)) == code


def test_gate_modes():
    lib = rola.load()
    p = rola.RolaParams()
    assert lib.rola_params_default(ctypes.byref(p)) == 0
    assert p.gate == 0                                 # ROLA_GATE_HEAD by default
    n = ctypes.c_size_t()
    for mode, code in ((0, 0), (1, 0), (2, 0), (3, 1), (-1, 1)):
        q = _params()
        q.gate = mode
        assert lib.rola_workspace_size(ctypes.byref(q), ctypes.byref(n)) == code
    # the gate does not change the workspace (gains or gate parameters are read in place)
    base = rola.workspace_size(_params())
    assert rola.workspace_size(_params(gate_per_token=True)) == base
    assert rola.workspace_size(_params(gate="proj")) == base


def test_block_size_must_be_64():
    p = _params()
    p.block = 32
    n = ctypes.c_size_t()
    assert rola.load().rola_workspace_size(ctypes.byref(p), ctypes.byref(n)) == 2


def test_workspace_size_grows_with_problem():
    a = rola.workspace_size(_params(N=1024))
    b = rola.workspace_size(_params(N=4096))
    assert 0 < a < b and a % 256 == 0


def test_plan_checks_workspace_without_touching_device():
    lib = rola.load()
    p = _params()
    need = rola.workspace_size(p)
    h = ctypes.c_void_p()
    assert lib.rola_plan(ctypes.byref(p), None, need, ctypes.byref(h)) == 3
    assert lib.rola_plan(ctypes.byref(p), ctypes.c_void_p(0x1000 + 16), need, ctypes.byref(h)) == 3
    assert lib.rola_plan(ctypes.byref(p), ctypes.c_void_p(0x100000), need - 1, ctypes.byref(h)) == 3
    # a well-formed (never dereferenced) address: plan creation is host-only
    assert lib.rola_plan(ctypes.byref(p), ctypes.c_void_p(0x100000), need, ctypes.byref(h)) == 0
    # null and misaligned tensors are rejected before any launch
    assert lib.rola_select_blocks(h, None, ctypes.c_void_p(0x2000), None) == 1
    assert lib.rola_select_blocks(h, ctypes.c_void_p(0x2008), ctypes.c_void_p(0x2000), None) == 1
    assert lib.rola_attend(h, *[ctypes.c_void_p(0x4000)] * 6, None) == 1   # out overlaps q
    assert lib.rola_set_debug(h, -1, 0) == 1
    # inspection calls reject missing buffers (and a missing plan) before any copy
    assert lib.rola_get_block_scores(h, None, ctypes.c_void_p(0x2000), None) == 1
    assert lib.rola_get_block_scores(None, ctypes.c_void_p(0x2000), ctypes.c_void_p(0x3000), None) == 1
    lib.rola_plan_destroy(h)


def test_status_strings():
    lib = rola.load()
    for c in range(7):
        assert lib.rola_status_string(c)
    assert lib.rola_status_string(0) == b"ok"


def test_fp8_configuration_host_rules():
    lib = rola.load()
    n = ctypes.c_size_t()
    # the e4m3 path is the head-dim-128 tcgen05 kernel only
    assert lib.rola_workspace_size(ctypes.byref(_params(d=64, dtype="fp8")), ctypes.byref(n)) == 2
    p8 = _params(d=128, r=32, dtype="fp8")
    pb = _params(d=128, r=32, dtype="bf16")
    # fp8 carries three one-byte copies and three scale arrays instead of the fp16 copy of v
    B, H, N, d = p8.B, p8.H, p8.N, p8.d
    nb = (N + 63) // 64
    extra = 3 * B * N * H * d + 3 * 4 * B * H * nb - 2 * B * N * H * d
    assert abs(rola.workspace_size(p8) - rola.workspace_size(pb) - extra) <= 6 * 256
    h = ctypes.c_void_p()
    need = rola.workspace_size(pb)
    assert lib.rola_plan(ctypes.byref(pb), ctypes.c_void_p(0x100000), need, ctypes.byref(h)) == 0
    bufs = [ctypes.c_void_p(0x200000 + 0x10000 * j) for j in range(6)]
    assert lib.rola_get_fp8_copies(h, *bufs, None) == 1      # not an fp8 plan
    lib.rola_plan_destroy(h)


def test_missing_library_fails_loudly_and_product_never_touches_the_oracle():
    """No fallback: without librola.so the binding raises; and neither the package nor its
    kernels import, link or read anything of the oracle (test infrastructure only)."""
    import subprocess
    import sys
    code = ("import sparse_rank_attention_b200 as r; r.LIB_PATH = '/nonexistent/librola.so'; r._lib = None\n"
            "try:\n    r.load()\nexcept RuntimeError as e:\n    print('raised', 'missing' in str(e))\n")
    p = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True, text=True, timeout=120)
    assert p.stdout.strip() == "raised True", p.stdout + p.stderr
    pkg = os.path.join(ROOT, "sparse_rank_attention_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f)).read()
                assert re.search(r"\boracle\b", text) is None, f"{f} mentions the oracle"
