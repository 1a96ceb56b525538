"""GPU parity of the backward (the next row f2: gradients of the RoLA forward) against the
oracle's backward, through the C ABI (rola_backward).

The oracle's backward is pinned against central differences of the forward oracle
(tests/test_oracle_backward.py).  Both sides take the kept-block lists of the forward as
fixed and differentiate the same function of the same input values (bf16 inputs enter both
as their exact values); the kernels compute in fp32 and the oracle in double, so the bound
is fp32 rounding over sums of up to k*64 terms, plus, at head dim 128 with bf16 inputs,
the state S from the tensor-core key/value pass (its feature operand as a bf16 hi + lo
pair, ~2^-16 relative): every element within 5e-4 of its tensor's RMS, and the whole
tensor within 5e-5 of it normwise.  The lists themselves are compared
bit for bit, and two calls must give identical bits (partial sums in a fixed order).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola
from rola_testlib import host_inputs, np32

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


CASES = [
    # the tiny fp32 configuration (1D grid)
    (synth.custom("bwd_tiny_f32", B=1, H=2, N=1024, d=64, r=16, topk=0.25, dtype="f32"), "head"),
    # bf16 at head dim 128: a ragged 40-token tail, a 3D grid, two batch entries
    (synth.custom("bwd_bf16_d128_b2", B=2, H=2, N=1000, d=128, r=32, topk=0.3, grid=(2, 4, 125)), "head"),
    (synth.custom("bwd_bf16_d128_token", B=1, H=3, N=777, d=128, r=32, topk=0.25, grid=(3, 7, 37)), "token"),
    (synth.custom("bwd_bf16_d128_proj", B=1, H=2, N=1000, d=128, r=16, topk=0.2), "proj"),
    (synth.custom("bwd_bf16_d64_r32", B=1, H=2, N=700, d=64, r=32, topk=0.4, grid=(7, 10, 10)), "head"),
    (synth.custom("bwd_f32_d128_tail1", B=2, H=1, N=129, d=128, r=32, topk=0.6, dtype="f32"), "token"),
    # several key-major passes per CTA wave: 128 blocks per head, 13 kept
    (synth.custom("bwd_bf16_d128_n8192", B=1, H=2, N=8192, d=128, r=32, topk=0.1, grid=(8, 32, 32)), "head"),
]


def _gain(w, gate, inp):
    if gate == "head":
        return inp["g"]
    if gate == "token":
        return synth.make_gate(w, seed=9, device="cuda")
    return synth.make_gate_proj(w, seed=9, device="cuda")


def _compare(name, got, want):
    got = got.astype(np.float64).reshape(-1)
    want = want.reshape(-1)
    rms = float(np.sqrt(np.mean(want ** 2))) or 1.0
    err = np.abs(got - want)
    worst = int(np.argmax(err))
    assert err[worst] <= 5e-4 * rms, f"{name}: |err| {err[worst]:.3e} at {worst} vs rms {rms:.3e}"
    nerr = float(np.sqrt(np.mean(err ** 2)))
    assert nerr <= 5e-5 * rms, f"{name}: normwise {nerr / rms:.3e}"


@pytest.mark.parametrize("w,gate", CASES, ids=[f"{w.name}-{g}" for w, g in CASES])
def test_backward_matches_oracle(w, gate):
    inp = synth.make_inputs(w, seed=5, device="cuda")
    g = _gain(w, gate, inp)
    dout = synth.make_dout(w, seed=6, device="cuda")
    plan = rola.Plan.for_workload(w, gate=gate)
    got = plan.backward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], g, dout)
    assert plan.poll_status() == 0
    again = plan.backward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], g, dout)
    torch.cuda.synchronize()
    for key in got:
        assert torch.equal(got[key], again[key]), f"{key} differs between two calls"
    h = host_inputs(inp)
    s = O.make_shape(w.B, w.H, w.N, w.d, w.r, w.topk, grid=w.grid, pairs=w.pairs, gate=gate)
    _, col = O.forward(s, h["q"], h["k"], h["v"], h["Wq"], h["Wk"], np32(g))
    np.testing.assert_array_equal(plan.block_lists().cpu().numpy(), col)
    want = O.backward(s, h["q"], h["k"], h["v"], h["Wq"], h["Wk"], np32(g), np32(dout).astype(np.float64), col)
    for key in ("dq", "dk", "dv", "dWq", "dWk", "dg"):
        _compare(f"{w.name}/{key}", np32(got[key]), want[key].reshape(np32(got[key]).shape))


def test_backward_rejects_bad_calls():
    w = synth.custom("bwd_args", B=1, H=2, N=256, d=128, r=32, topk=0.5)
    inp = synth.make_inputs(w, seed=1, device="cuda")
    dout = synth.make_dout(w, seed=2, device="cuda")
    plan = rola.Plan.for_workload(w)
    lib = rola.load()
    grads = plan.backward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], dout)
    ws = plan.bwd_workspace
    p = lambda t: rola._ptr(t)  # noqa: E731
    args = [p(inp[n]) for n in ("q", "k", "v", "Wq", "Wk", "g")] + [p(dout)]
    outs = [p(grads[n]) for n in ("dq", "dk", "dv", "dWq", "dWk", "dg")]
    st = rola._stream(None)
    assert lib.rola_backward(plan._h, *args, *outs, p(ws), ws.numel(), st) == 0
    assert lib.rola_backward(plan._h, *args, *outs, p(ws), ws.numel() - 256, st) == 3   # scratch too small
    bad = list(outs)
    bad[0] = p(inp["q"])                                                             # dq over q
    assert lib.rola_backward(plan._h, *args, *bad, p(ws), ws.numel(), st) == 1
    bad = list(outs)
    bad[1] = outs[0]                                                                 # dk over dq
    assert lib.rola_backward(plan._h, *args, *bad, p(ws), ws.numel(), st) == 1
    assert lib.rola_backward(plan._h, *args[:6], rola._ptr(None), *outs, p(ws), ws.numel(), st) == 1
    w8 = synth.custom("bwd_fp8", B=1, H=2, N=256, d=128, r=32, topk=0.5, dtype="fp8")
    n = rola.ctypes.c_size_t()
    assert lib.rola_backward_workspace_size(rola.ctypes.byref(rola.Plan.for_workload(w8).params),
                                            rola.ctypes.byref(n)) == 2
    assert plan.poll_status() == 0


@pytest.mark.parametrize("wname", ["wan21_14b_480p"])
def test_backward_at_full_size_on_sampled_heads_and_blocks(wname):
    """The whole backward at a Wan shape, checked on two heads: their dWq, dWk, dg (summed
    over every token) and, on seeded query and key blocks including the ragged tail, dq and
    dk, dv, against the oracle's sampled backward (pinned to its whole backward)."""
    w = synth.WORKLOADS[wname]
    inp = synth.make_inputs(w, seed=11, device="cuda")
    dout = synth.make_dout(w, seed=12, device="cuda")
    plan = rola.Plan.for_workload(w)
    got = plan.backward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], dout)
    assert plan.poll_status() == 0
    col = plan.block_lists().cpu().numpy()
    rng = np.random.default_rng(3)
    heads = sorted(rng.choice(w.H, size=2, replace=False).tolist())
    nb = plan.nb
    blocks = lambda: [0, nb - 1] + rng.choice(np.arange(1, nb - 1), size=2, replace=False).tolist()  # noqa: E731
    qb = [(0, h, i) for h in heads for i in blocks()]
    kb = [(0, h, j) for h in heads for j in blocks()]
    h = host_inputs(inp)
    s = O.make_shape(w.B, w.H, w.N, w.d, w.r, w.topk, grid=w.grid, pairs=w.pairs)
    smp = O.backward_sample(s, h["q"], h["k"], h["v"], h["Wq"], h["Wk"], h["g"],
                            np32(dout).astype(np.float64), col, heads, qb, kb)
    def rows(t, blist):
        out = np.zeros((len(blist), 64, w.d))
        for e, (b, hh, i) in enumerate(blist):
            n = min(w.N, i * 64 + 64) - i * 64
            out[e, :n] = np32(t[b, i * 64:i * 64 + n, hh])
        return out
    _compare("dq", rows(got["dq"], qb), smp["dq"])
    _compare("dk", rows(got["dk"], kb), smp["dk"])
    _compare("dv", rows(got["dv"], kb), smp["dv"])
    _compare("dWq", np32(got["dWq"])[heads], smp["dWq"])
    _compare("dWk", np32(got["dWk"])[heads], smp["dWk"])
    _compare("dg", np32(got["dg"])[heads], smp["dg"])


@pytest.mark.parametrize("top", [1.5, 40.0])
def test_backward_with_peaked_softmax_rows(top):
    """Key blocks scaled up along the sequence (the inputs that send forward tiles to the
    careful pass): the softmax rows are peaked and their logits span a wide range; the
    backward takes each row's exact lse, so it must hold the same bound.  With keys up to 41x
    larger, later blocks score far above the first pair of a row, so the tensor-core row
    statistics hand those query tiles to the block-by-block kernel."""
    w = synth.custom("bwd_bf16_rising", B=1, H=2, N=4096, d=128, r=32, topk=0.25, grid=(4, 16, 64))
    inp = synth.make_inputs(w, seed=7, device="cuda")
    nb = w.nb
    scale = 1.0 + top * torch.arange(nb, device="cuda", dtype=torch.float32) / nb
    inp["k"] = (inp["k"].float() * scale.repeat_interleave(64)[: w.N].view(1, w.N, 1, 1)).to(inp["k"].dtype)
    dout = synth.make_dout(w, seed=8, device="cuda")
    plan = rola.Plan.for_workload(w)
    got = plan.backward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], dout)
    assert plan.poll_status() == 0
    h = host_inputs(inp)
    s = O.make_shape(w.B, w.H, w.N, w.d, w.r, w.topk, grid=w.grid, pairs=w.pairs)
    _, col = O.forward(s, h["q"], h["k"], h["v"], h["Wq"], h["Wk"], h["g"])
    np.testing.assert_array_equal(plan.block_lists().cpu().numpy(), col)
    want = O.backward(s, h["q"], h["k"], h["v"], h["Wq"], h["Wk"], h["g"], np32(dout).astype(np.float64), col)
    for key in ("dq", "dk", "dv", "dWq", "dWk", "dg"):
        _compare(f"{w.name}/{key}", np32(got[key]), want[key].reshape(np32(got[key]).shape))
