"""The tensor-core block scores that prune the selection, against the error bound the exact
top-k relies on.

The kept lists are decided on exact fp32 scores (checked bit for bit against the oracle in
test_gpu_parity.py and test_zz_no_alloc.py); the scores s~ (three tf32 products of a hi/lo
split) only rule blocks out, with |s~ - s| <= 2^-14 |qbar_i| |kbar_j| (+ terms below 2^-116)
taken as the bound.  Here the error of s~ against the scores of the same pooled means in
double must stay within half of that (2^-15 |qbar_i| |kbar_j|; the split's own terms are
below 2^-18), so the margin the bound assumes for the tensor cores' fp32 accumulation holds
on the hardware, and the key-block norms must be the norms.
"""
import numpy as np
import pytest
import torch

import synth
import sparse_rank_attention_b200 as rola

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


CASES = [
    synth.custom("scores_bf16_d128", B=1, H=3, N=5000, d=128, r=32, topk=0.1, grid=(5, 10, 100)),
    synth.custom("scores_f32_d64", B=2, H=2, N=1000, d=64, r=16, topk=0.25, dtype="f32"),
    synth.custom("scores_bf16_small", B=1, H=2, N=200, d=128, r=32, topk=0.5),
]


@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_tensor_core_scores_within_half_the_bound(w):
    inp = synth.make_inputs(w, seed=21, device="cuda")
    # spread the key norms over two orders of magnitude
    kscale = torch.logspace(-1, 1, w.N, device="cuda").view(1, w.N, 1, 1)
    inp["k"] = (inp["k"].float() * kscale).to(inp["k"].dtype)
    plan = rola.Plan.for_workload(w)
    plan.select_blocks(inp["q"], inp["k"])
    assert plan.poll_status() == 0
    qb, kb = (t.cpu().double().numpy() for t in plan.pooled())
    sc, kn = (t.cpu().double().numpy() for t in plan.block_scores())
    exact = np.einsum("bhic,bhjc->bhij", qb, kb)
    qn = np.sqrt((qb ** 2).sum(-1))
    kn64 = np.sqrt((kb ** 2).sum(-1))
    np.testing.assert_allclose(kn, kn64, rtol=1e-6, atol=0)
    bound = 2.0 ** -15 * qn[..., :, None] * kn64[..., None, :] + 2.0 ** -116
    err = np.abs(sc - exact)
    worst = np.unravel_index(np.argmax(err / bound), err.shape)
    assert np.all(err <= bound), f"{w.name}: |s~ - s| {err[worst]:.3e} > {bound[worst]:.3e} at {worst}"


def test_selection_with_ties_everywhere_takes_the_exact_path():
    """Every key block equal: no tensor-core score can tell them apart, every block is a
    candidate, and the kept lists are the first k blocks of every row."""
    w = synth.custom("scores_all_tied", B=1, H=2, N=64 * 300, d=128, r=32, topk=0.1)
    inp = synth.make_inputs(w, seed=3, device="cuda")
    inp["k"] = inp["k"][:, :64].repeat(1, 300, 1, 1).contiguous()
    plan = rola.Plan.for_workload(w)
    plan.select_blocks(inp["q"], inp["k"])
    assert plan.poll_status() == 0
    lists = plan.block_lists().cpu().numpy()
    want = np.broadcast_to(np.arange(plan.k, dtype=np.int32), lists.shape)
    np.testing.assert_array_equal(lists, want)
