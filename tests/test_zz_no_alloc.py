"""The allocation-free block selection (rola_select_blocks_noalloc) against the planned one
and against the oracle.

That entry point serves callers that cannot allocate device memory at the point of the
call and have no workspace to lend (a host framework whose pool owns all device memory,
or a latency-critical path that cannot take cudaMalloc's implicit synchronisation).  It
keeps its scratch in a fixed array inside the library, shared by every call, so two calls
in a row must both reproduce the planned path's block lists exactly, and those lists must
equal the oracle's.  The bf16, fp8 (whose lists come from the bf16 inputs) and fp32
head-dim-64 configurations each take their own pooling route through it.  This file is
collected last on purpose."""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola
from rola_testlib import host_inputs, shape_of

pytestmark = pytest.mark.gpu

ROLA_ERR_WORKSPACE = 3
ROLA_ERR_INVALID_ARG = 1


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


CASES = [
    synth.custom("noalloc_bf16", B=1, H=4, N=4096, d=128, r=32, topk=0.1, grid=(1, 4, 1024)),
    synth.custom("noalloc_fp8", B=1, H=3, N=3000, d=128, r=32, topk=0.1, grid=(2, 30, 50), dtype="fp8"),
    synth.custom("noalloc_f32_d64", B=2, H=2, N=1000, d=64, r=16, topk=0.25, dtype="f32"),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_noalloc_selection_matches_planned_selection_twice(w):
    params = rola.make_params(w.B, w.H, w.N, w.d, w.r, w.topk, w.grid, dtype=w.dtype)
    s = shape_of(w)
    for seed in (11, 12):                       # two calls in a row, different inputs
        inp = synth.make_inputs(w, seed=seed, device="cuda")
        plan = rola.Plan.for_workload(w)
        plan.select_blocks(inp["q"], inp["k"])
        want = plan.block_lists()
        got = torch.full_like(want, -1)
        assert rola.select_blocks_noalloc(params, inp["q"], inp["k"], got) == 0
        torch.cuda.synchronize()
        assert torch.equal(got, want)           # block lists are bit-exact
        h = host_inputs(inp)
        col, *_ = O.select(s, O.pool(s, h["q"]), O.pool(s, h["k"]))
        np.testing.assert_array_equal(got.cpu().numpy(), col)


def test_noalloc_rejects_problems_beyond_its_scratch():
    w = synth.WORKLOADS["wan21_14b_720p"]
    params = rola.make_params(w.B, w.H, w.N, w.d, w.r, w.topk, w.grid, dtype=w.dtype)
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    col = torch.empty(16, dtype=torch.int32, device="cuda")
    assert rola.select_blocks_noalloc(params, q, q, col) == ROLA_ERR_WORKSPACE


def test_noalloc_rejects_lists_overlapping_an_input():
    w = CASES[0]
    params = rola.make_params(w.B, w.H, w.N, w.d, w.r, w.topk, w.grid, dtype=w.dtype)
    inp = synth.make_inputs(w, seed=1, device="cuda")
    alias = inp["k"].view(torch.int32)          # the lists would overwrite k
    assert rola.select_blocks_noalloc(params, inp["q"], inp["k"], alias) == ROLA_ERR_INVALID_ARG
