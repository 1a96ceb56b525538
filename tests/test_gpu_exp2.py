"""The softmax exponentials of the head-dim-128 attention kernels against exp2 in double.

Attention weights are P = exp(s - m) ("SparkDiffusion ..." page, section "RoLA: Preserving
Global Context at Extreme Sparsity", the block-sparse softmax branch); the kernels write
them as 2^x with x = (s - m) log2(e) <= 0.  Most come from the special-function unit's
ex2.approx; the e4m3 path takes a quarter from a cubic polynomial on the FMA pipe, whose
range reduction (round to n, splice n into the exponent field) and clamp at -125 are what
this file checks, over a dense sweep of x in [-125, 0] with the integer and half-integer
points, the clamp and the special values."""
import numpy as np
import pytest
import torch

import sparse_rank_attention_b200 as rola

pytestmark = pytest.mark.gpu

POLY_REL = 7.8e-5          # the fit's stated relative error bound on [-125, 0]
APPROX_REL = 2.0 ** -21    # ex2.approx: about 2 ulp of fp32


def _sweep():
    dense = np.linspace(-125.0, 0.0, 2_000_001)
    ints = np.arange(-125, 1, dtype=np.float64)
    halves = ints[:-1] + 0.5
    near = np.concatenate([ints + e for e in (-1e-6, 1e-6, -0.49999, 0.49999)])
    x = np.concatenate([dense, ints, halves, near])
    return x[(x >= -125.0) & (x <= 0.0)].astype(np.float32)


@pytest.mark.parametrize("mode,bound", [(0, APPROX_REL), (1, POLY_REL)])
def test_exp2_relative_error_over_the_softmax_range(mode, bound):
    x32 = _sweep()
    y = rola.eval_exp2(torch.from_numpy(x32).cuda(), mode).cpu().numpy().astype(np.float64)
    ref = np.exp2(x32.astype(np.float64))
    rel = np.abs(y - ref) / ref
    worst = int(np.argmax(rel))
    assert rel[worst] <= bound, (mode, float(x32[worst]), float(rel[worst]))
    # no bias: the mean signed error is well inside the bound
    assert abs(float(np.mean((y - ref) / ref))) < bound / 4


def test_exp2_special_values():
    x = torch.tensor([0.0, -0.0, -1.0, -0.5, -124.5, -125.0, -126.0, -200.0, -float("inf"),
                      float("nan")], device="cuda")
    a = rola.eval_exp2(x, 0).cpu()
    p = rola.eval_exp2(x, 1).cpu()
    assert a[0] == 1.0 and a[1] == 1.0 and a[2] == 0.5
    assert a[8] == 0.0                                        # 2^-inf = 0 (masked keys)
    assert torch.isnan(a[9])
    assert abs(float(p[0]) - 1.0) <= POLY_REL and abs(float(p[2]) - 0.5) <= 0.5 * POLY_REL
    two_m125 = 2.0 ** -125
    for i in (5, 6, 7, 8, 9):                                 # clamped: 2^-125
        assert abs(float(p[i]) - two_m125) <= POLY_REL * two_m125, (i, float(p[i]))


def test_exp2_rejects_bad_arguments():
    lib = rola.load()
    x = torch.zeros(4, device="cuda")
    assert lib.rola_eval_exp2(x.data_ptr(), x.data_ptr(), 4, 2, None) == 1
    assert lib.rola_eval_exp2(x.data_ptr(), x.data_ptr(), -1, 0, None) == 1
    assert lib.rola_eval_exp2(None, x.data_ptr(), 4, 0, None) == 1
    assert lib.rola_eval_exp2(None, None, 0, 0, None) == 0
