"""Failure detection on the GPU without faulting it: a bounded device-side wait that
runs out reports ROLA_ERR_DEVICE_TIMEOUT through the status word and the context stays
usable; non-finite inputs are reported as ROLA_ERR_RANGE."""
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


def _run(plan, inp, out=None):
    return plan.forward(inp["q"], inp["k"], inp["v"], inp["Wq"], inp["Wk"], inp["g"], out)


def test_stalled_wait_reports_timeout_and_recovers():
    w = synth.custom("stall", B=1, H=2, N=1024, d=128, r=32, topk=0.25)
    inp = synth.make_inputs(w, seed=5, device="cuda")
    plan = rola.Plan.for_workload(w)
    ref = _run(plan, inp)
    assert plan.poll_status() == 0
    plan.set_debug(rola.ROLA_DEBUG_STALL_WAIT, 2000)      # a barrier nothing arrives on, 2 ms
    _run(plan, inp, torch.empty_like(ref))
    assert plan.poll_status() == 5                          # ROLA_ERR_DEVICE_TIMEOUT
    assert plan.poll_status() == 0                          # reading clears it
    plan.set_debug(0, 0)
    again = _run(plan, inp)
    assert plan.poll_status() == 0
    torch.cuda.synchronize()
    assert torch.equal(again, ref)


@pytest.mark.parametrize("d", [128, 64])
def test_non_finite_value_is_reported(d):
    w = synth.custom("range", B=1, H=2, N=512, d=d, r=32, topk=0.25)
    inp = synth.make_inputs(w, seed=6, device="cuda")
    inp["v"][0, 100, 1, 7] = float("inf")
    plan = rola.Plan.for_workload(w)
    _run(plan, inp)
    assert plan.poll_status() == 7                          # ROLA_ERR_RANGE
