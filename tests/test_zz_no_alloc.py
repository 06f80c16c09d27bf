"""skv_attn_fwd_noalloc: the forward + merge entry point for callers that
cannot allocate device memory (a plugin handed only tensor pointers by a host
framework that owns the device memory, or latency-critical code that must not
call cudaMalloc/cudaFree). Its workspace is a 32 MiB static device array
inside the library. Checked through the C ABI against the workspace-based
entry points (skv_attn_fwd + skv_lse_merge), with the forward tolerances used
by the other parity tests, on two calls in a row. This file is collected
last on purpose."""
import numpy as np
import pytest
import torch

from oracle import attention as A
from split_kv_block_b200 import skv, synth

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 2e-2, 1e-3


def _inputs(prob, seed):
    q, k, v, _ = synth.make_tensors(prob, seed=seed, backward=False)
    return q.cuda(), k.cuda(), v.cuda()


def _reference(plan, q, k, v):
    ws = skv.alloc_workspace(plan)
    o, lse = skv.forward(plan, q, k, v, ws)
    assert skv.skv_status(ws) == 0
    return o, lse


def _noalloc(plan, q, k, v):
    p = plan.problem
    o = torch.full((p.num_tokens_q, p.num_q_heads, p.head_dim), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((p.num_tokens_q, p.num_q_heads), float("nan"), dtype=torch.float32, device="cuda")
    skv.skv_attn_fwd_noalloc(plan, q, k, v, o, lse)
    torch.cuda.synchronize()
    return o, lse


def _close(a, b):
    (o1, l1), (o2, l2) = a, b
    assert torch.isfinite(o1.float()).all() and torch.isfinite(l1).all()
    assert float((o1.float() - o2.float()).abs().max()) <= O_TOL
    assert float((l1 - l2).abs().max()) <= LSE_TOL


def test_noalloc_matches_workspace_path_two_calls():
    # two different problems back to back: the second call must not see the
    # first call's leftovers in the shared scratch
    prob1 = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0)
    prob2 = synth.small_problem([1001, 777], [[1000, 3, 555], [777, 1]], block_q=16, chunk_kv=256,
                                num_partitions=3, hq=8, hkv=2, d=128)
    for prob, seed in ((prob1, 0), (prob2, 1)):
        plan = skv.skv_plan(prob)
        assert plan.sizes.ws_fwd_bytes <= skv.SKV_NOALLOC_SCRATCH_BYTES
        q, k, v = _inputs(prob, seed)
        _close(_noalloc(plan, q, k, v), _reference(plan, q, k, v))
    # and the same problem twice in a row
    plan = skv.skv_plan(prob1)
    q, k, v = _inputs(prob1, 0)
    ref = _reference(plan, q, k, v)
    _close(_noalloc(plan, q, k, v), ref)
    _close(_noalloc(plan, q, k, v), ref)


def test_noalloc_matches_the_oracle_and_reports_ok():
    """The tiny workload straight against the fp64 oracle, and the status
    word of the call read back through skv_noalloc_status (no allocation)."""
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=2)
    plan = skv.skv_plan(prob)
    qc, kc, vc, _ = synth.make_tensors(prob, seed=2, backward=False)
    o, lse = _noalloc(plan, qc.cuda(), kc.cuda(), vc.cuda())
    assert skv.skv_noalloc_status() == 0
    O_ref, L_ref = A.attention_forward(prob, qc, kc, vc)
    assert float((o.cpu().double() - O_ref).abs().max()) <= O_TOL
    assert float((lse.cpu().double() - L_ref).abs().max()) <= LSE_TOL


def test_noalloc_rejects_problems_beyond_the_scratch():
    prob = synth.make_problem(synth.WORKLOADS["ctx32k_fwd"], seed=0)
    plan = skv.skv_plan(prob)
    assert plan.sizes.ws_fwd_bytes > skv.SKV_NOALLOC_SCRATCH_BYTES
    q, k, v = _inputs(prob, 0)
    o = torch.empty(prob.num_tokens_q, prob.num_q_heads, prob.head_dim, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(prob.num_tokens_q, prob.num_q_heads, dtype=torch.float32, device="cuda")
    with pytest.raises(skv.SkvError) as e:
        skv.skv_attn_fwd_noalloc(plan, q, k, v, o, lse)
    assert e.value.code == 8
