"""Failure detection of the device-side waits, tested without a GPU fault:
a bounded mbarrier wait that nothing completes gives up after its limit and
leaves SKV_ETIMEOUT in the workspace status word; the context stays usable
(a full forward + backward afterwards runs clean)."""
import pytest
import torch

from split_kv_block_b200 import skv, synth

pytestmark = pytest.mark.gpu

SKV_OK, SKV_EINVAL, SKV_ETIMEOUT = 0, 1, 6


def test_wait_that_nobody_completes_times_out_and_reports():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    skv.skv_wait_selftest(ws, 1_000_000, arrive=True)   # 1 ms limit, phase completed first
    assert skv.skv_status(ws) == SKV_OK
    skv.skv_wait_selftest(ws, 1_000_000, arrive=False)  # nothing completes the phase
    assert skv.skv_status(ws) == SKV_ETIMEOUT
    assert "time" in skv.lib().skv_strerror(SKV_ETIMEOUT).decode().lower()
    skv.skv_wait_selftest(ws, 1_000_000, arrive=True)   # the status word is cleared per call
    assert skv.skv_status(ws) == SKV_OK


def test_context_usable_after_a_timeout():
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    skv.skv_wait_selftest(ws, 2_000_000, arrive=False)
    assert skv.skv_status(ws) == SKV_ETIMEOUT
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=2)
    q, k, v, do = [t.cuda() for t in synth.make_tensors(prob, seed=2, backward=True)]
    plan = skv.skv_plan(prob)
    w2 = skv.alloc_workspace(plan)
    o, lse = skv.forward(plan, q, k, v, w2)
    skv.backward(plan, q, k, v, o, lse, do, w2)
    assert skv.skv_status(w2) == SKV_OK
    assert torch.isfinite(o.float()).all()


def test_invalid_arguments_are_refused_before_launch():
    ws = torch.zeros(512, dtype=torch.uint8, device="cuda")
    with pytest.raises(skv.SkvError) as e:
        skv.skv_wait_selftest(ws[1:], 1000, arrive=True)     # misaligned
    assert e.value.code == SKV_EINVAL
    with pytest.raises(skv.SkvError) as e:
        skv.skv_wait_selftest(ws, 0, arrive=True)           # no limit
    assert e.value.code == SKV_EINVAL
