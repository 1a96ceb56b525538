"""GPU parity of the input-dependent gates against the CPU oracle.

The README's sparse-finetuning section on the SparkDiffusion page names gate_proj and
gate_bias among RoLA's parameters without fixing their form.  Two gates are built:
  * "token": the gain that scales the linear branch is read per token and head, g[B, N, H]
    (the values any gate computed outside the operator would give);
  * "proj": the gain is computed inside from the query, g = sigmoid(q . gate_proj_h +
    gate_bias_h), with g holding gate_proj [H, d] and gate_bias [H].
Everything else is the per-head computation.  Each compute path (tcgen05 bf16 and fp8 at
head dim 128, the head-dim-64 path, the fp32 path) is compared in full with the oracle at
the same tolerances as the per-head tests, and a per-token gate equal to the per-head gains
must reproduce the per-head output bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola
from rola_testlib import check_out, check_out_fp8, gather_blocks, host_inputs, np32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


def _gate_shape(w, gate="token"):
    return O.make_shape(w.B, w.H, w.N, w.d, w.r, w.topk, grid=w.grid, pairs=w.pairs, gate=gate)


CASES = [
    synth.custom("gate_bf16_d128_b2", B=2, H=2, N=1000, d=128, r=32, topk=0.25, grid=(2, 4, 125)),
    synth.custom("gate_fp8_d128", B=1, H=2, N=1000, d=128, r=32, topk=0.25, dtype="fp8"),
    synth.custom("gate_bf16_d64_3d", B=2, H=3, N=777, d=64, r=16, topk=0.3, grid=(3, 7, 37)),
    synth.custom("gate_f32_tail1", B=2, H=1, N=129, d=64, r=16, topk=0.6, dtype="f32"),
]


@pytest.mark.parametrize("gate_kind", ["token", "proj"])
@pytest.mark.parametrize("w", CASES, ids=[w.name for w in CASES])
def test_input_dependent_gate_matches_oracle(w, gate_kind):
    inp = synth.make_inputs(w, seed=4, device="cuda")
    if gate_kind == "token":
        gate = synth.make_gate(w, seed=9, device="cuda")
    else:
        gate = synth.make_gate_proj(w, seed=9, device="cuda")
    plan = rola.Plan.for_workload(w, gate=gate_kind)
    out = torch.empty_like(inp["q"])
    plan.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], gate, out)
    assert plan.poll_status() == 0
    h = host_inputs(inp)
    want, col = O.forward(_gate_shape(w, gate_kind), h["q"], h["k"], h["v"], h["Wq"], h["Wk"],
                          np32(gate))
    np.testing.assert_array_equal(plan.block_lists().cpu().numpy(), col)
    got = np32(out).astype(np.float64)
    if w.dtype == "fp8":
        blocks = np.array([(b, hh, i) for b in range(w.B) for hh in range(w.H) for i in range(w.nb)],
                          dtype=np.int32)
        g_rows, valid = gather_blocks(got, blocks, w.N)
        w_rows, _ = gather_blocks(want, blocks, w.N)
        norm, worst = check_out_fp8(g_rows, w_rows, valid, w.name)
        print(f"PARITY {w.name} {gate_kind} normwise={norm:.3e} worst_block={worst:.3e}")
    else:
        err, rms = check_out(got, want, w.dtype, w.name)
        print(f"PARITY {w.name} {gate_kind} max_err={err:.3e} rms={rms}")


def test_per_token_gate_equal_to_head_gains_is_bit_identical():
    w = synth.custom("gate_bcast_bf16", B=1, H=3, N=1536, d=128, r=32, topk=0.2, grid=(2, 6, 128))
    inp = synth.make_inputs(w, seed=6, device="cuda")
    per_head = rola.Plan.for_workload(w)
    per_token = rola.Plan.for_workload(w, gate_per_token=True)
    out_h = per_head.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"])
    g_tok = inp["g"].view(1, 1, w.H).expand(w.B, w.N, w.H).contiguous()
    out_t = per_token.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], g_tok)
    assert per_head.poll_status() == 0 and per_token.poll_status() == 0
    assert torch.equal(out_h, out_t)


def test_projected_gate_with_zero_weights_equals_the_head_gains_of_its_bias():
    """gate_proj = 0: every token's gain is sigmoid(gate_bias_h); with gate_bias = logit(g_h)
    the output equals the per-head output with gains g_h (up to the fp32 sigmoid)."""
    w = synth.custom("gate_proj_zero_w", B=1, H=3, N=1536, d=128, r=32, topk=0.2, grid=(2, 6, 128))
    inp = synth.make_inputs(w, seed=6, device="cuda")
    gh = inp["g"]
    params = torch.cat([torch.zeros(w.H * w.d, device="cuda"), torch.log(gh / (1 - gh))]).contiguous()
    out_h = rola.Plan.for_workload(w).forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], gh)
    out_p = rola.Plan.for_workload(w, gate="proj").forward(inp["q"], inp["k"], inp["v"], inp["Wq"],
                                                            inp["Wk"], params)
    torch.cuda.synchronize()
    err = (out_h.float() - out_p.float()).abs().max().item()
    rms = out_h.float().pow(2).mean().sqrt().item()
    assert err <= 1e-2 * rms, (err, rms)
