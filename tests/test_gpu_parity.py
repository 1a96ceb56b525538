"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Small cases are compared in full (every output element, every block list, the
pooled means and the linear state).  The Wan-shaped workloads are compared at full
size on every block list, pooled mean and state entry, and on a seeded sample of
query blocks (always including the ragged tail block) for the outputs.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola
from rola_testlib import (check_out, gather_blocks, host_inputs, np32, run_gpu, sample_blocks,
                          shape_of)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


def _state_tol(dtype):
    return 1e-4 if dtype == "f32" else 1e-2


def _compare_full(w, seed=0):
    inp = synth.make_inputs(w, seed=seed, device="cuda")
    res = run_gpu(w, inp)
    assert res["status"] == 0
    h = host_inputs(inp)
    s = shape_of(w)
    qbar, kbar = O.pool(s, h["q"]), O.pool(s, h["k"])
    np.testing.assert_array_equal(res["qbar"], qbar)
    np.testing.assert_array_equal(res["kbar"], kbar)
    col, *_ = O.select(s, qbar, kbar)
    np.testing.assert_array_equal(res["col"], col)
    S, z = O.linear_state(s, h["k"], h["v"], h["Wk"])
    rmsS = np.sqrt(np.mean(S ** 2))
    assert np.abs(res["S"] - S).max() <= _state_tol(w.dtype) * rmsS
    assert np.abs(res["z"] - z).max() <= _state_tol(w.dtype) * 1e-1 * np.abs(z).max()
    out, _ = O.forward(s, h["q"], h["k"], h["v"], h["Wq"], h["Wk"], h["g"])
    r = check_out(np32(res["out"]).astype(np.float64), out, w.dtype, w.name)
    print(f"PARITY {w.name} max_err={r[0]:.3e} rms={r[1]}")
    return r


def test_tiny_f32_full():
    _compare_full(synth.WORKLOADS["tiny_f32_h2_n1024"])


SMALL = [
    synth.custom("bf16_ragged40", B=1, H=2, N=1000, d=128, r=32, topk=0.25),
    synth.custom("bf16_b2_h3_d64_3d", B=2, H=3, N=777, d=64, r=16, topk=0.3, grid=(3, 7, 37)),
    synth.custom("bf16_tail1", B=1, H=1, N=321, d=128, r=16, topk=0.5),
    synth.custom("bf16_single_block", B=1, H=2, N=48, d=128, r=32, topk=0.1),
    synth.custom("bf16_tail56_3d", B=1, H=2, N=4152, d=128, r=32, topk=0.1, grid=(2, 4, 519)),
    synth.custom("bf16_keep_all", B=1, H=2, N=640, d=64, r=32, topk=1.0, grid=(2, 5, 64)),
    synth.custom("bf16_keep_one", B=1, H=2, N=2048, d=128, r=32, topk=0.01, grid=(2, 2, 512)),
    synth.custom("bf16_pairs_custom", B=1, H=2, N=1536, d=128, r=32, topk=0.2, grid=(4, 6, 64),
                 pairs=(2, 6, 8)),
    synth.custom("bf16_block_offsets", B=1, H=2, N=2048, d=128, r=32, topk=0.125,
                 dist="block_offset"),
    synth.custom("f32_d128_r32_3d", B=1, H=2, N=900, d=128, r=32, topk=0.3, grid=(3, 5, 60),
                 dtype="f32"),
    synth.custom("f32_tail1", B=2, H=1, N=129, d=64, r=16, topk=0.6, dtype="f32"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_small_full(w):
    _compare_full(w, seed=1)


def test_exact_ties_keep_lower_block_index():
    """Duplicated key blocks give exactly equal block scores: both sides keep the lower index."""
    w = synth.custom("ties", B=1, H=2, N=1024, d=128, r=32, topk=0.25)
    inp = synth.make_inputs(w, seed=3, device="cuda")
    k = inp["k"]
    for src, dst in ((2, 9), (2, 13), (5, 6), (0, 15)):
        k[:, 64 * dst:64 * dst + 64] = k[:, 64 * src:64 * src + 64]
    res = run_gpu(w, inp)
    h = host_inputs(inp)
    s = shape_of(w)
    col, kth, nxt, _ = O.select(s, O.pool(s, h["q"]), O.pool(s, h["k"]))
    assert np.any(kth == nxt)          # the planted ties reach the selection boundary
    np.testing.assert_array_equal(res["col"], col)


def test_run_to_run_bitwise_identical():
    w = synth.custom("det", B=1, H=4, N=8192, d=128, r=32, topk=0.1, grid=(2, 64, 64))
    inp = synth.make_inputs(w, seed=4, device="cuda")
    plan = rola.Plan.for_workload(w)
    a = plan.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"])
    Sa, za = plan.state()
    b = plan.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"])
    Sb, zb = plan.state()
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(Sa, Sb) and torch.equal(za, zb)


def _compare_sampled(w, n_heads=3, n_blocks=12, seed=0):
    inp = synth.make_inputs(w, seed=seed, device="cuda")
    res = run_gpu(w, inp)
    assert res["status"] == 0
    out_gpu = np32(res["out"])
    h = host_inputs(inp)
    del inp
    torch.cuda.empty_cache()
    s = shape_of(w)
    qbar, kbar = O.pool(s, h["q"]), O.pool(s, h["k"])
    np.testing.assert_array_equal(res["qbar"], qbar)
    np.testing.assert_array_equal(res["kbar"], kbar)
    col, *_ = O.select(s, qbar, kbar)
    np.testing.assert_array_equal(res["col"], col)
    S, z = O.linear_state(s, h["k"], h["v"], h["Wk"])
    assert np.abs(res["S"] - S).max() <= _state_tol(w.dtype) * np.sqrt(np.mean(S ** 2))
    blocks = sample_blocks(w, n_heads, n_blocks, seed)
    _, _, want = O.attend_blocks(s, h["q"], h["k"], h["v"], h["Wq"], h["g"], col, S, z, blocks)
    got, valid = gather_blocks(out_gpu, blocks, w.N)
    r = check_out(got[valid], want[valid], w.dtype, w.name)
    print(f"PARITY {w.name} max_err={r[0]:.3e} rms={r[1]}")
    return r


@pytest.mark.parametrize("name", ["wan21_1p3b_480p", "wan21_14b_480p", "wan21_14b_720p",
                                  "wan21_14b_480p_dense_g0", "wan21_14b_480p_topk0.25",
                                  "wan21_14b_480p_cfg_b2"])
def test_wan_shapes_sampled(name):
    _compare_sampled(synth.WORKLOADS[name])


def test_longest_sequence_accepted_sampled():
    """The largest block count the library accepts (6000 blocks: N = 384 000 tokens, one
    head): every block list, mean and state entry, and sampled query blocks of the output."""
    w = synth.custom("max_blocks_6000", B=1, H=1, N=6000 * 64, d=128, r=32, topk=0.01,
                     grid=(20, 100, 192))
    assert w.nb == 6000
    _compare_sampled(w, n_heads=1, n_blocks=16, seed=3)


def _rising_keys(inp, w, top=6.0):
    """Scales key block j by 1 + top * j / nb: later kept blocks score far above the first
    pair of each row, so the fast attention pass must hand tiles to the careful pass."""
    nb = w.nb
    scale = 1.0 + top * torch.arange(nb, device=inp["k"].device, dtype=torch.float32) / nb
    per_tok = scale.repeat_interleave(64)[: w.N].view(1, w.N, 1, 1)
    inp["k"] = (inp["k"].float() * per_tok).to(inp["k"].dtype)
    return inp


def test_careful_pass_recomputes_overflowing_tiles():
    w = synth.custom("bf16_rising", B=1, H=2, N=4096, d=128, r=32, topk=0.25, grid=(4, 16, 64))
    inp = _rising_keys(synth.make_inputs(w, seed=7, device="cuda"), w, top=1.5)
    res = run_gpu(w, inp)
    assert res["status"] == 0
    assert res["plan"].attend_redo_count() > 0      # the careful pass ran on some tiles
    h = host_inputs(inp)
    out, _ = O.forward(shape_of(w), h["q"], h["k"], h["v"], h["Wq"], h["Wk"], h["g"])
    r = check_out(np32(res["out"]).astype(np.float64), out, w.dtype, w.name)
    print(f"PARITY {w.name} redo={res['plan'].attend_redo_count()} max_err={r[0]:.3e} rms={r[1]}")


def test_fast_pass_alone_on_wan_like_inputs():
    w = synth.custom("bf16_wan_like", B=1, H=2, N=4152, d=128, r=32, topk=0.1, grid=(2, 4, 519))
    res = run_gpu(w, synth.make_inputs(w, seed=1, device="cuda"))
    assert res["status"] == 0 and res["plan"].attend_redo_count() == 0
