"""Pins of the oracle's backward (the next row f2: gradients of the RoLA forward).

The backward is derived by the chain rule from the forward's definition ("SparkDiffusion
..." page, section "RoLA: Preserving Global Context at Extreme Sparsity": the block-sparse
softmax branch plus the low-rank linear branch with rotary positions; README
sparse-finetuning section: proj_q, proj_k, gate_proj, gate_bias).  Each gradient is held
against central differences of the forward oracle (already pinned on its own): for
L = sum(dout * out), dL/dx ~ (L(x + h) - L(x - h)) / 2h with h = 2^-14, exact in float32
for these inputs, and the kept-block lists checked unchanged by each step.  Every term of
the derivation (each branch, the normaliser, phi', the rotation's transpose, each gain
form) moves some element, so a dropped term or a wrong sign fails here."""
import numpy as np
import pytest

import oracle

H_STEP = 2.0 ** -14


def _problem(gate, seed=0):
    rng = np.random.default_rng(seed)
    B, H, N, d, r = 1, 2, 200, 16, 8
    grid = (2, 10, 10)
    s = oracle.make_shape(B, H, N, d, r, 0.5, grid=grid, gate=gate)
    nb = oracle.num_blocks(N)
    off = rng.normal(0, 1.0, (B, nb, H, d))
    def act():
        x = rng.normal(0, 1, (B, N, H, d)) + np.repeat(off, 64, axis=1)[:, :N]
        return x.astype(np.float32)
    q, k, v = act(), act(), act()
    Wq = (rng.normal(0, 1, (H, d, r)) / np.sqrt(d)).astype(np.float32)
    Wk = (rng.normal(0, 1, (H, d, r)) / np.sqrt(d)).astype(np.float32)
    if gate == "head":
        g = rng.uniform(0.1, 1.0, H)
    elif gate == "token":
        g = rng.uniform(0.0, 1.0, B * N * H)
    else:
        g = np.concatenate([rng.normal(0, 1 / np.sqrt(d), H * d), rng.uniform(-0.5, 0.5, H)])
    dout = rng.normal(0, 1, (B, N, H, d))
    return s, dict(q=q, k=k, v=v, Wq=Wq, Wk=Wk, g=g), dout


def _loss(s, inp, dout):
    out, col = oracle.forward(s, inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"])
    return float(np.sum(dout * out)), col


GRAD_OF = {"q": "dq", "k": "dk", "v": "dv", "Wq": "dWq", "Wk": "dWk", "g": "dg"}


@pytest.mark.parametrize("gate", ["head", "token", "proj"])
def test_backward_matches_central_differences(gate):
    s, inp, dout = _problem(gate)
    _, col = _loss(s, inp, dout)
    grads = oracle.backward(s, inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], dout, col)
    rng = np.random.default_rng(1)
    for name, gname in GRAD_OF.items():
        x = inp[name]
        flat = x.reshape(-1)
        picks = rng.choice(flat.size, size=min(12, flat.size), replace=False)
        for e in picks:
            saved = flat[e]
            flat[e] = saved + H_STEP
            lp, colp = _loss(s, inp, dout)
            flat[e] = saved - H_STEP
            lm, colm = _loss(s, inp, dout)
            flat[e] = saved
            assert np.array_equal(colp, col) and np.array_equal(colm, col), (name, e)
            fd = (lp - lm) / (2 * H_STEP)
            an = grads[gname].reshape(-1)[e]
            assert abs(fd - an) <= 2e-5 * max(1.0, abs(an)), (gate, name, int(e), fd, an)


def test_backward_zero_gain_has_no_linear_gradient():
    """g = 0: the linear branch drops out, so Wq and Wk get no gradient and dg is the
    dout-weighted sum of the linear output (central differences cover its value)."""
    s, inp, dout = _problem("head", seed=3)
    inp["g"] = np.zeros(s.H)
    _, col = _loss(s, inp, dout)
    gr = oracle.backward(s, inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], dout, col)
    assert np.all(gr["dWq"] == 0) and np.all(gr["dWk"] == 0)
    assert np.all(gr["dg"] != 0)


def test_backward_is_linear_in_dout():
    s, inp, dout = _problem("head", seed=4)
    _, col = _loss(s, inp, dout)
    a = oracle.backward(s, inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], dout, col)
    b = oracle.backward(s, inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], 3.0 * dout, col)
    for key in a:
        np.testing.assert_allclose(b[key], 3.0 * a[key], rtol=1e-12, atol=1e-12)


def test_sampled_backward_equals_the_whole_one():
    """The sampled form (for problems too large for the whole backward) gives, on the listed
    heads and blocks, what the whole backward gives (B = 2: dWq, dWk, dg sum over the batch)."""
    rng = np.random.default_rng(7)
    B, H, N, d, r = 2, 3, 300, 16, 8
    s = oracle.make_shape(B, H, N, d, r, 0.4, grid=(3, 10, 10))
    q, k, v = (rng.normal(0, 1, (B, N, H, d)).astype(np.float32) for _ in range(3))
    Wq, Wk = (rng.normal(0, 1 / np.sqrt(d), (H, d, r)).astype(np.float32) for _ in range(2))
    g = rng.uniform(0.1, 1.0, H)
    dout = rng.normal(0, 1, (B, N, H, d))
    _, col = oracle.forward(s, q, k, v, Wq, Wk, g)
    full = oracle.backward(s, q, k, v, Wq, Wk, g, dout, col)
    heads = [0, 2]
    qb = [(0, 0, 1), (1, 2, 4), (1, 0, 0)]          # block 4 is the 44-token tail
    kb = [(1, 2, 2), (0, 0, 4), (0, 2, 0)]
    smp = oracle.backward_sample(s, q, k, v, Wq, Wk, g, dout, col, heads, qb, kb)
    for e, (b, h, i) in enumerate(qb):
        rows = slice(i * 64, min(N, i * 64 + 64))
        n = rows.stop - rows.start
        np.testing.assert_allclose(smp["dq"][e, :n], full["dq"][b, rows, h], rtol=1e-10, atol=1e-12)
        assert np.all(smp["dq"][e, n:] == 0)
    for e, (b, h, j) in enumerate(kb):
        rows = slice(j * 64, min(N, j * 64 + 64))
        n = rows.stop - rows.start
        np.testing.assert_allclose(smp["dk"][e, :n], full["dk"][b, rows, h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(smp["dv"][e, :n], full["dv"][b, rows, h], rtol=1e-10, atol=1e-12)
    for t, h in enumerate(heads):
        np.testing.assert_allclose(smp["dWq"][t], full["dWq"][h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(smp["dWk"][t], full["dWk"][h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(smp["dg"][t], full["dg"][h], rtol=1e-10, atol=1e-12)
