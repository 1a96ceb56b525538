"""The allocation-free block selection (rola_select_blocks_noalloc) against the planned one.

That entry point serves callers that cannot allocate device memory at the point of the
call and have no workspace to lend (a host framework whose pool owns all device memory,
or a latency-critical path that cannot take cudaMalloc's implicit synchronisation).  It
keeps its scratch in a fixed array inside the library, shared by every call, so two calls
in a row must both reproduce the planned path's block lists exactly.  This file is
collected last on purpose."""
import pytest
import torch

import synth
import sparse_rank_attention_b200 as rola

pytestmark = pytest.mark.gpu

ROLA_ERR_WORKSPACE = 3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


def test_noalloc_selection_matches_planned_selection_twice():
    w = synth.custom("noalloc", B=1, H=4, N=4096, d=128, r=32, topk=0.1, grid=(1, 4, 1024))
    params = rola.make_params(w.B, w.H, w.N, w.d, w.r, w.topk, w.grid, dtype=w.dtype)
    for seed in (11, 12):                       # two calls in a row, different inputs
        inp = synth.make_inputs(w, seed=seed, device="cuda")
        plan = rola.Plan.for_workload(w)
        plan.select_blocks(inp["q"], inp["k"])
        want = plan.block_lists()
        got = torch.full_like(want, -1)
        assert rola.select_blocks_noalloc(params, inp["q"], inp["k"], got) == 0
        torch.cuda.synchronize()
        assert torch.equal(got, want)           # block lists are bit-exact


def test_noalloc_rejects_problems_beyond_its_scratch():
    w = synth.WORKLOADS["wan21_14b_720p"]
    params = rola.make_params(w.B, w.H, w.N, w.d, w.r, w.topk, w.grid, dtype=w.dtype)
    q = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    col = torch.empty(16, dtype=torch.int32, device="cuda")
    assert rola.select_blocks_noalloc(params, q, q, col) == ROLA_ERR_WORKSPACE
