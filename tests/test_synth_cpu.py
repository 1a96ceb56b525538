"""The seeded input generators shared by the parity tests and the benchmark (CPU): the same
seed gives the same tensors, different seeds different ones, with the stated shapes, types
and ranges."""
import torch

import synth


def test_inputs_are_reproducible_and_shaped():
    w = synth.custom("synth_check", B=2, H=3, N=200, d=64, r=16, topk=0.5, grid=(2, 4, 25))
    a = synth.make_inputs(w, seed=7)
    b = synth.make_inputs(w, seed=7)
    c = synth.make_inputs(w, seed=8)
    for name in ("q", "k", "v", "Wq", "Wk", "g"):
        assert torch.equal(a[name], b[name]), name
    assert not torch.equal(a["q"], c["q"])
    assert a["q"].shape == (2, 200, 3, 64) and a["q"].dtype == torch.bfloat16
    assert a["Wq"].shape == (3, 64, 16) and a["g"].shape == (3,) and a["g"].dtype == torch.float32
    assert bool(((a["g"] >= 0.1) & (a["g"] <= 1.0)).all())


def test_gate_is_reproducible_per_token_and_in_range():
    w = synth.custom("gate_check", B=2, H=3, N=130, d=64, r=16, topk=0.5)
    g1, g2, g3 = synth.make_gate(w, seed=1), synth.make_gate(w, seed=1), synth.make_gate(w, seed=2)
    assert g1.shape == (2, 130, 3) and g1.dtype == torch.float32
    assert torch.equal(g1, g2) and not torch.equal(g1, g3)
    assert bool(((g1 >= 0) & (g1 < 1)).all())
    assert g1.std() > 0.2                               # varies across tokens


def test_cfg_batch_workload_is_the_480p_shape_with_two_entries():
    w, base = synth.WORKLOADS["wan21_14b_480p_cfg_b2"], synth.WORKLOADS["wan21_14b_480p"]
    assert (w.B, w.H, w.N, w.d, w.r, w.topk, w.grid) == (2, base.H, base.N, base.d, base.r, base.topk,
                                                          base.grid)


def test_gate_projection_parameters_are_reproducible_and_shaped():
    w = synth.custom("gp", B=1, H=3, N=100, d=64, r=16)
    a = synth.make_gate_proj(w, seed=2)
    b = synth.make_gate_proj(w, seed=2)
    assert a.shape == (w.H * (w.d + 1),) and a.dtype == torch.float32
    assert torch.equal(a, b)
    bias = a[w.H * w.d:]
    assert torch.all(bias.abs() <= 0.5)
    assert 0.5 / w.d ** 0.5 < a[:w.H * w.d].std() < 2.0 / w.d ** 0.5
