"""GPU parity of the fp8-e4m3 configuration against the CPU oracle.

* The block lists and pooled means come from the bf16 inputs: bit-exact, as for bf16.
* The e4m3 copies of q, k, v and their per-(b, h, block) scales: bit-exact against the
  oracle's quantiser (the codes are integer results decided in fp32, as in the kernels).
* The output: normwise within 6e-2 of RMS against the oracle on the bf16 inputs (the
  operator's tolerance), and, as a tighter diagnostic, within 3e-2 of RMS against the
  oracle run on the dequantised q, k, v (what is left there is the e4m3 rounding of the
  softmax weights and fp32 accumulation).
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth
import sparse_rank_attention_b200 as rola
from rola_testlib import (check_out_fp8, gather_blocks, host_inputs, np32, run_gpu, sample_blocks,
                          shape_of)

pytestmark = pytest.mark.gpu
DIAG_TOL = 3e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    rola.load()


def _all_blocks(w):
    return np.array([(b, h, i) for b in range(w.B) for h in range(w.H) for i in range(w.nb)],
                    dtype=np.int32)


def _check(w, seed, blocks=None, copies_full=True, modify=None):
    inp = synth.make_inputs(w, seed=seed, device="cuda")
    if modify is not None:
        inp = modify(inp)
    res = run_gpu(w, inp)
    assert res["status"] == 0
    (q8, k8, v8), (sq, sk, sv) = res["plan"].fp8_copies()
    q8, k8, v8 = (t.cpu().numpy() for t in (q8, k8, v8))
    sq, sk, sv = (t.cpu().numpy() for t in (sq, sk, sv))
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
    deq = {}
    for name, codes, scales in (("q", q8, sq), ("k", k8, sk), ("v", v8, sv)):
        want_codes, want_scales = O.quantize_blocks(s, h[name])
        np.testing.assert_array_equal(scales, want_scales, err_msg=f"{name} scales")
        np.testing.assert_array_equal(codes, want_codes, err_msg=f"{name} e4m3 codes")
        deq[name] = O.dequantize_blocks(s, want_codes, want_scales)
    S, z = O.linear_state(s, h["k"], h["v"], h["Wk"])
    assert np.abs(res["S"] - S).max() <= 1e-2 * np.sqrt(np.mean(S ** 2))
    blocks = _all_blocks(w) if blocks is None else blocks
    sp, _, want = O.attend_blocks(s, h["q"], h["k"], h["v"], h["Wq"], h["g"], col, S, z, blocks)
    sp_q, _, _ = O.attend_blocks(s, deq["q"], deq["k"], deq["v"], h["Wq"], h["g"], col, S, z, blocks)
    want_q = want - sp + sp_q          # sparse branch on the dequantised inputs, same linear branch
    got, valid = gather_blocks(out_gpu, blocks, w.N)
    norm, worst = check_out_fp8(got, want, valid, w.name)
    diag, _ = check_out_fp8(got, want_q, valid, w.name + " (dequantised inputs)", tol=DIAG_TOL)
    print(f"PARITY {w.name} normwise={norm:.3e} worst_block={worst:.3e} vs_dequantised={diag:.3e}")
    return res


SMALL = [
    synth.custom("fp8_ragged40", B=1, H=2, N=1000, d=128, r=32, topk=0.25, dtype="fp8"),
    synth.custom("fp8_tail1_r16", B=1, H=1, N=321, d=128, r=16, topk=0.5, dtype="fp8"),
    synth.custom("fp8_single_block", B=1, H=2, N=48, d=128, r=32, topk=0.1, dtype="fp8"),
    synth.custom("fp8_tail56_3d", B=2, H=2, N=4152, d=128, r=32, topk=0.1, grid=(2, 4, 519),
                 dtype="fp8"),
    synth.custom("fp8_keep_all", B=1, H=2, N=640, d=128, r=32, topk=1.0, grid=(2, 5, 64), dtype="fp8"),
    synth.custom("fp8_keep_one", B=1, H=2, N=2048, d=128, r=32, topk=0.01, grid=(2, 2, 512),
                 dtype="fp8"),
    synth.custom("fp8_block_offsets", B=1, H=2, N=2048, d=128, r=32, topk=0.125, dist="block_offset",
                 dtype="fp8"),
    # more than 3 x 148 tiles: each persistent CTA runs several tiles, across heads and batches
    synth.custom("fp8_multitile_b2_tail54", B=2, H=4, N=7990, d=128, r=32, topk=0.1, grid=(2, 17, 235),
                 dtype="fp8"),
]


@pytest.mark.parametrize("w", SMALL, ids=[w.name for w in SMALL])
def test_fp8_small_full(w):
    _check(w, seed=2)


def test_fp8_zero_block_scale_is_one():
    """An all-zero 64-token block of v quantises with scale 1 and contributes zeros."""
    w = synth.custom("fp8_zero_block", B=1, H=2, N=1024, d=128, r=32, topk=0.5, dtype="fp8")
    inp = synth.make_inputs(w, seed=5, device="cuda")
    inp["v"][:, 128:192] = 0
    inp["q"][:, 320:384, 1] = 0
    plan = rola.Plan.for_workload(w)
    plan.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"])
    (q8, _, v8), (sq, _, sv) = plan.fp8_copies()
    assert plan.poll_status() == 0
    assert torch.all(sv[0, :, 2] == 1.0) and torch.all(v8[0, 128:192] == 0)
    assert sq[0, 1, 5] == 1.0 and torch.all(q8[0, 320:384, 1] == 0)


def test_fp8_wan_720p_sampled():
    w = synth.WORKLOADS["wan21_14b_720p_fp8"]
    _check(w, seed=0, blocks=sample_blocks(w, 4, 64, 0))


def test_fp8_careful_pass_recomputes_overflowing_tiles():
    """Later key blocks scaled up (by at most 1.8x): scores rise more than 8 (log2) above a
    tile's first pair, so its e4m3 weights would saturate and the careful pass redoes it."""
    from test_gpu_parity import _rising_keys
    w = synth.custom("fp8_rising", B=1, H=2, N=4096, d=128, r=32, topk=0.25, grid=(4, 16, 64), dtype="fp8")
    res = _check(w, seed=7, modify=lambda inp: _rising_keys(inp, w, top=0.8))
    assert res["plan"].attend_redo_count() > 0
