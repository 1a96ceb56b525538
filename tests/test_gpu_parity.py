"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Small cases are compared in full (every output element, every block list, the
pooled means and the linear state).  Two of them have more than three query-block
tiles per SM (1024 and 1000 tiles over 148 persistent CTAs), so every CTA of the
tcgen05 attention kernel walks several tiles and crosses head (and batch) boundaries
while compared element by element.  The Wan-shaped workloads, including every point of
the 14B-480P sparsity sweep, are compared at full size on every block list, pooled mean
and state entry, and on a seeded sample of at least 4 heads x 64 query blocks (always
including the first and the ragged tail block) for the outputs.
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
    # more than 3 x 148 tiles: each persistent CTA runs several tiles, across heads
    synth.custom("bf16_multitile_h8", B=1, H=8, N=8192, d=128, r=32, topk=0.1, grid=(2, 64, 64)),
    synth.custom("bf16_multitile_b2_tail54", B=2, H=4, N=7990, d=128, r=32, topk=0.1,
                 grid=(2, 17, 235)),
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


def _compare_sampled(w, n_heads=4, n_blocks=64, seed=0):
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


# every Wan shape, the whole 14B-480P sparsity sweep (topk 0.03 / 0.05 / 0.1 / 0.25 / 1 with
# per-head gains, and 1 with g = 0), the B = 2 classifier-free-guidance batch, the I2V
# grids (portrait, square with a 5-token last block, 49 frames) and Wan2.2-A14B at topk 0.1
@pytest.mark.parametrize("name", ["wan21_1p3b_480p", "wan21_14b_480p", "wan21_14b_720p",
                                  "wan21_14b_480p_topk0.03", "wan21_14b_480p_topk0.1",
                                  "wan21_14b_480p_topk0.25", "wan21_14b_480p_topk1",
                                  "wan21_14b_480p_dense_g0", "wan21_14b_480p_cfg_b2",
                                  "wan21_14b_i2v_480p_portrait", "wan21_14b_i2v_480p_square",
                                  "wan21_14b_i2v_480p_49f", "wan22_a14b_480p", "wan22_a14b_720p"])
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


def _wide_range_v(inp, w):
    """v spread over the whole bf16 range: blocks scaled by 1e6, 1e-6 and 1e30 (values
    outside fp16's range both ways), the rest left as drawn."""
    v = inp["v"].float()
    for blk, f in ((1, 1e6), (3, 1e-6), (6, 1e30), (9, 1e-30), (12, 3e4)):
        v[:, 64 * blk:64 * blk + 64] *= f
    inp["v"] = v.to(inp["v"].dtype)
    return inp


@pytest.mark.parametrize("g_const", [0.0, None], ids=["sparse_only", "with_linear"])
@pytest.mark.parametrize("d", [128, 64])
def test_v_over_the_whole_bf16_range(d, g_const):
    """Every finite bf16 v is accepted: the fp16 copy of v carries one power-of-two exponent
    per block, applied back inside the attention (in the careful pass where a row's kept
    blocks differ).  Compared in full with the oracle; with g = 0 the output is the sparse
    branch alone, so each query block's check sees its own kept blocks' scale (the linear
    branch, over all keys, would otherwise carry the 1e30 blocks into every row)."""
    w = synth.custom(f"bf16_wide_v_d{d}", B=1, H=2, N=1000, d=d, r=32, topk=0.5, grid=(1, 8, 125),
                     g_const=g_const)
    inp = _wide_range_v(synth.make_inputs(w, seed=8, device="cuda"), w)
    res = run_gpu(w, inp)
    assert res["status"] == 0
    if d == 128:
        assert res["plan"].attend_redo_count() > 0   # rows mixing exponents took the careful pass
    h = host_inputs(inp)
    out, col = O.forward(shape_of(w), h["q"], h["k"], h["v"], h["Wq"], h["Wk"], h["g"])
    np.testing.assert_array_equal(res["col"], col)
    got = np32(res["out"]).astype(np.float64)
    # rows differ by up to 1e60 in magnitude here: the tolerance is taken per query block
    # (2e-2 of the block's own RMS plus half an ulp), so small rows are held to their scale
    for b in range(w.B):
        for hh in range(w.H):
            for i in range(w.nb):
                n0, n1 = 64 * i, min(w.N, 64 * i + 64)
                check_out(got[b, n0:n1, hh], out[b, n0:n1, hh], "bf16", f"{w.name} h{hh} block {i}")
