"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Tolerances (bf16 inputs, fp32 accumulation): forward output max-abs <= 2e-2,
LSE max-abs <= 1e-3, gradients relative Frobenius <= 1e-2 per tensor.
Heads are independent, so where the oracle would be slow it runs on a subset
of kv-head groups (exact for those heads).
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from split_kv_block_b200 import skv, synth

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL, GRAD_TOL = 2e-2, 1e-3, 1e-2


def _dev(*ts):
    return [t.cuda() if t is not None else None for t in ts]


def _heads_subset(prob, groups):
    G = prob.num_q_heads // prob.num_kv_heads
    qh = [g * G + i for g in groups for i in range(G)]
    return qh, list(groups), prob.replace(num_q_heads=len(qh), num_kv_heads=len(groups))


def _rel_fro(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm().clamp_min(1e-30))


def run_gpu(prob, q, k, v, do=None, policy=skv.SKV_PLAN_LPT, fused=True):
    plan = skv.skv_plan(prob, policy)
    qd, kd, vd, dod = _dev(q, k, v, do)
    ws = skv.alloc_workspace(plan)
    o, lse = skv.forward(plan, qd, kd, vd, ws, fused=fused)
    assert skv.skv_status(ws) == 0
    grads = None
    if do is not None:
        grads = skv.backward(plan, qd, kd, vd, o, lse, dod, ws)
        assert skv.skv_status(ws) == 0
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu(), (None if grads is None else [g.cpu() for g in grads]), plan


def check_forward(prob, q, k, v, o, lse, groups=None):
    if groups is not None:
        qh, kh, sub = _heads_subset(prob, groups)
        q, k, v = q[:, qh].contiguous(), k[:, kh].contiguous(), v[:, kh].contiguous()
        o, lse, prob = o[:, qh], lse[:, qh], sub
    O_ref, L_ref = A.attention_forward(prob, q, k, v)
    err_o = float((o.double() - O_ref).abs().max()) if o.numel() else 0.0
    # rows that attend no key (possible under a block-sparse mask): LSE = -inf on both sides
    none = torch.isneginf(L_ref)
    assert torch.equal(torch.isneginf(lse), none), "rows without keys differ"
    lse, L_ref = lse.double()[~none], L_ref[~none]
    err_l = float((lse.double() - L_ref).abs().max()) if lse.numel() else 0.0
    assert err_o <= O_TOL, f"O max-abs {err_o}"
    assert err_l <= LSE_TOL, f"LSE max-abs {err_l}"
    return O_ref, L_ref, err_o, err_l


def check_backward(prob, q, k, v, do, grads, groups=None):
    dq, dk, dv = grads
    if groups is not None:
        qh, kh, sub = _heads_subset(prob, groups)
        q, k, v, do = q[:, qh].contiguous(), k[:, kh].contiguous(), v[:, kh].contiguous(), do[:, qh].contiguous()
        dq, dk, dv, prob = dq[:, qh], dk[:, kh], dv[:, kh], sub
    O_ref, L_ref = A.attention_forward(prob, q, k, v)
    rq, rk, rv = A.attention_backward(prob, q, k, v, O_ref, L_ref, do)
    errs = (_rel_fro(dq, rq), _rel_fro(dk, rk), _rel_fro(dv, rv))
    assert max(errs) <= GRAD_TOL, f"rel fro dq/dk/dv {errs}"
    # keys no query sees: exactly zero
    for b in range(prob.num_samples):
        j0, j1 = int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])
        amax = int(prob.anchors[j0:j1].max()) if j1 > j0 else 0
        k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
        assert torch.all(dk[k0 + amax:k1] == 0) and torch.all(dv[k0 + amax:k1] == 0)
    return errs


def _case(prob, seed=0, backward=True, policy=skv.SKV_PLAN_LPT, groups=None, fused=True):
    q, k, v, do = synth.make_tensors(prob, seed=seed, backward=backward)
    o, lse, grads, plan = run_gpu(prob, q, k, v, do, policy, fused)
    check_forward(prob, q, k, v, o, lse, groups)
    if backward:
        check_backward(prob, q, k, v, do, grads, groups)
    return plan


def test_tiny_4k_forward_and_backward():
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0)
    _case(prob)


def test_plan_buffer_is_free_once_the_call_returns():
    """The forward and the backward take the plan's device section through the
    library's own staging slot (copied there during the call, read by the upload
    kernel when the stream reaches it), so the caller may overwrite its plan
    buffer as soon as a call returns, before the GPU has run that call."""
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0)
    q, k, v, do = synth.make_tensors(prob, seed=0, backward=True)
    qd, kd, vd, dod = _dev(q, k, v, do)
    plan = skv.skv_plan(prob, skv.SKV_PLAN_LPT)
    orig = plan.buf.copy()
    ws = skv.alloc_workspace(plan)
    Nq, Hq, d = prob.num_tokens_q, prob.num_q_heads, prob.head_dim
    o = torch.empty(Nq, Hq, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(Nq, Hq, dtype=torch.float32, device="cuda")
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    stream = torch.cuda.current_stream()
    torch.cuda.synchronize()
    torch.cuda._sleep(20_000_000)  # about 10 ms: the call is enqueued long before the stream reaches it
    skv.skv_attn_fwd(plan, qd, kd, vd, ws, stream)
    plan.buf[:] = 0xA5
    torch.cuda.synchronize()
    plan.buf[:] = orig
    skv.skv_lse_merge(plan, ws, o, lse, stream)
    torch.cuda._sleep(20_000_000)
    skv.skv_attn_bwd(plan, qd, kd, vd, o, lse, dod, dq, dk, dv, ws, stream)
    plan.buf[:] = 0x5A
    torch.cuda.synchronize()
    plan.buf[:] = orig
    assert skv.skv_status(ws) == 0
    check_forward(prob, q, k, v, o.cpu(), lse.cpu())
    check_backward(prob, q, k, v, do, [dq.cpu(), dk.cpu(), dv.cpu()])


def test_tiny_4k_static_plan():
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=1)
    _case(prob, seed=1, policy=skv.SKV_PLAN_STATIC)


@pytest.mark.parametrize("d", [64, 128])
def test_random_ragged_problems(d):
    rng = np.random.default_rng(100 + d)
    for i in range(6):
        prob = synth.random_small_problem(rng, max_len=900, max_anchors=7, d=d,
                                          heads=((4, 1), (8, 2), (4, 4), (8, 1), (16, 2), (2, 2)))
        _case(prob, seed=i, policy=skv.SKV_PLAN_LPT if i % 3 else skv.SKV_PLAN_STATIC, fused=i % 2 == 0)


def test_edge_anchors():
    """a = 1, a = L, duplicates, unsorted anchors, block_q = 1."""
    prob = synth.small_problem([517, 260], [[1, 517, 517, 3, 200], [260, 1, 129]], block_q=1, chunk_kv=128,
                               sub_chunks=2, num_partitions=5, hq=8, hkv=2, d=128)
    _case(prob)


def test_partitions_exceed_items_and_single_partition():
    prob = synth.small_problem([300], [[299, 10, 150]], block_q=16, chunk_kv=256, num_partitions=32, hq=4, hkv=1,
                               d=64)
    _case(prob)
    _case(prob.replace(num_partitions=1))


def test_sample_without_anchors():
    prob = synth.small_problem([400, 333, 128], [[390], [], [128, 5]], block_q=16, chunk_kv=128, num_partitions=3,
                               hq=4, hkv=1, d=64)
    _case(prob)


def test_ragged_tiles_many_samples():
    """Odd anchor counts (query tiles half empty), chunk not a multiple of the
    key tile, context lengths not multiples of anything."""
    prob = synth.small_problem([1001, 777, 1500], [[1000, 3, 555], [777], [1, 1499, 700, 64, 1200]], block_q=16,
                               chunk_kv=320, num_partitions=4, hq=8, hkv=2, d=128)
    _case(prob, seed=3)


def test_ctx32k_two_groups():
    """The 32K workload at full size; oracle on 2 of the 8 kv-head groups."""
    prob = synth.make_problem(synth.WORKLOADS["ctx32k"], seed=0)
    _case(prob, groups=(0, 5))


def _one_sample(prob, b, q, k, v, do, o, lse, grads):
    """Sub-problem of sample b alone (its tokens, its context) with the matching
    slices of inputs and GPU outputs; exact, samples are independent."""
    S = prob.block_q
    j0, j1 = int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])
    k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
    t0, t1 = j0 * S, j1 * S
    sub = prob.replace(ctx_offsets=np.array([0, k1 - k0], dtype=np.int64),
                       anchor_offsets=np.array([0, j1 - j0], dtype=np.int32), anchors=prob.anchors[j0:j1].copy())
    dq, dk, dv = grads
    return (sub, q[t0:t1], k[k0:k1], v[k0:k1], do[t0:t1], o[t0:t1], lse[t0:t1],
            (dq[t0:t1], dk[k0:k1], dv[k0:k1]))


def test_ctx128k_full_size_one_group():
    """The 128K Beta(5,1) workload at full size with 4 key sub-chunks per chunk
    (the <= 1% imbalance granularity); oracle on one kv-head group."""
    prob = synth.make_problem(synth.WORKLOADS["ctx128k"], seed=0, sub_chunks=4)
    _case(prob, groups=(3,))


def test_ctx128k_full_size_chunk_items_one_group():
    """The 128K Beta(5,1) workload at full size with whole-chunk items
    (sub_chunks = 1, 4096-key items: the plan the benchmark times); oracle on
    one kv-head group."""
    prob = synth.make_problem(synth.WORKLOADS["ctx128k"], seed=0, sub_chunks=1)
    assert prob.sub_chunks == 1
    _case(prob, groups=(6,))


def test_batch8_full_size_one_sample_one_group():
    """The batched workload (8 samples, contexts 8K-256K) at full size with
    fresh anchors; oracle on the longest sample and on a mid-sized one, one
    kv-head group each."""
    w = synth.WORKLOADS["batch8_logu"]
    prob = synth.redraw_anchors(synth.make_problem(w, seed=0), w, seed=11)
    q, k, v, do = synth.make_tensors(prob, seed=0, backward=True)
    o, lse, grads, plan = run_gpu(prob, q, k, v, do)
    lens = np.diff(prob.ctx_offsets)
    order = np.argsort(lens)
    for b, g in ((int(order[-1]), 2), (int(order[len(lens) // 2]), 6)):  # the longest, a mid-sized sample
        sub, qs, ks, vs, dos, os_, ls, gs = _one_sample(prob, b, q, k, v, do, o, lse, grads)
        check_forward(sub, qs, ks, vs, os_, ls, groups=(g,))
        check_backward(sub, qs, ks, vs, dos, gs, groups=(g,))


def test_dead_key_gradients_are_written_zero():
    """Keys past every anchor of their sample get dK = dV = 0 written by the
    backward itself (the outputs start as NaN here), in every sample."""
    prob = synth.small_problem([700, 513, 900], [[300, 2], [513], [64, 450, 10]], block_q=16, chunk_kv=256,
                               num_partitions=3, hq=8, hkv=2, d=128)
    q, k, v, do = synth.make_tensors(prob, seed=5, backward=True)
    plan = skv.skv_plan(prob)
    qd, kd, vd, dod = _dev(q, k, v, do)
    ws = skv.alloc_workspace(plan)
    o, lse = skv.forward(plan, qd, kd, vd, ws)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(vd, float("nan"))
    skv.skv_attn_bwd(plan, qd, kd, vd, o, lse, dod, dq, dk, dv, ws)
    assert skv.skv_status(ws) == 0
    torch.cuda.synchronize()
    check_backward(prob, q, k, v, do, (dq.cpu(), dk.cpu(), dv.cpu()))
    assert not torch.isnan(dk).any() and not torch.isnan(dv).any() and not torch.isnan(dq).any()


@pytest.mark.parametrize("name", ["tiny_4k", "ctx32k_fwd"])
def test_merge_in_the_forward_tail_equals_the_merge_kernel(name):
    """skv_attn_fwd_merged (the merge in the forward kernel's tail) against
    skv_attn_fwd + skv_lse_merge: the same partials merged by the same
    arithmetic in the same order, so o and lse are bitwise equal; both
    within tolerance of the oracle on the tiny workload."""
    prob = synth.make_problem(synth.WORKLOADS[name], seed=4)
    q, k, v, _ = synth.make_tensors(prob, seed=4, backward=False)
    plan = skv.skv_plan(prob)
    qd, kd, vd = _dev(q, k, v)
    ws = skv.alloc_workspace(plan)
    o1, l1 = skv.forward(plan, qd, kd, vd, ws, fused=True)
    assert skv.skv_status(ws) == 0
    o2, l2 = skv.forward(plan, qd, kd, vd, ws, fused=False)
    assert skv.skv_status(ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))
    if name == "tiny_4k":
        check_forward(prob, q, k, v, o1.cpu(), l1.cpu())


@pytest.mark.parametrize("fused", [False, True])
def test_bf16_partials(fused):
    """Plans with SKV_PLAN_PARTIALS_BF16: the same forward tolerances against
    the oracle (the partial outputs are convex combinations of bf16 values,
    rounded once more), through the merge kernel and through the merge in
    the forward's tail; head_dim 64 and 128, ragged tiles, the 32K workload."""
    flag = skv.SKV_PLAN_PARTIALS_BF16
    cases = [(synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=3), None),
             (synth.small_problem([1001, 777, 1500], [[1000, 3, 555], [777], [1, 1499, 700, 64, 1200]],
                                  block_q=16, chunk_kv=320, num_partitions=4, hq=8, hkv=2, d=128), None),
             (synth.make_problem(synth.WORKLOADS["ctx32k_fwd"], seed=1), (2, 7))]
    for prob, groups in cases:
        q, k, v, _ = synth.make_tensors(prob, seed=3, backward=False)
        o, lse, _, _ = run_gpu(prob, q, k, v, None, skv.SKV_PLAN_LPT | flag, fused)
        check_forward(prob, q, k, v, o, lse, groups)


def test_tile_cost_plans():
    """Plans placed on the executed-tile cost run the same kernels: the tiny
    workload and a ragged problem, forward and backward."""
    _case(synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=2), seed=2, policy=skv.SKV_PLAN_LPT_TILES)
    prob = synth.small_problem([1001, 777, 1500], [[1000, 3, 555], [777], [1, 1499, 700, 64, 1200]], block_q=16,
                               chunk_kv=320, num_partitions=4, hq=8, hkv=2, d=128)
    _case(prob, seed=6, policy=skv.SKV_PLAN_LPT_TILES)


def test_partition_queue_plans():
    """SKV_PLAN_PARTITION_QUEUES (one work queue per partition, CTAs stealing
    from the next queue when theirs is empty): forward and backward against
    the oracle, head_dim 64 and 128, ragged tiles, both merges, and the 128K
    workload on one kv-head group."""
    flag = skv.SKV_PLAN_PARTITION_QUEUES
    _case(synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=4), seed=4, policy=skv.SKV_PLAN_LPT | flag)
    prob = synth.small_problem([1001, 777, 1500], [[1000, 3, 555], [777], [1, 1499, 700, 64, 1200]], block_q=16,
                               chunk_kv=320, num_partitions=4, hq=8, hkv=2, d=128)
    _case(prob, seed=7, policy=skv.SKV_PLAN_LPT | flag)
    _case(prob, seed=7, policy=skv.SKV_PLAN_STATIC | flag, fused=False)
    _case(synth.make_problem(synth.WORKLOADS["ctx128k"], seed=0), seed=0, policy=skv.SKV_PLAN_LPT | flag,
          groups=(5,))


def test_queue_modes_compute_the_same_bits():
    """The work queues only decide which CTA runs a unit and when: every
    forward unit's partial, hence the merged O and LSE, and the deterministic
    backward's dQ, dK and dV are the same bits with one queue and with one
    queue per partition (ctx32k, and a ragged three-sample problem)."""
    for prob in (synth.make_problem(synth.WORKLOADS["ctx32k"], seed=1),
                 synth.small_problem([1001, 777, 1500], [[1000, 3, 555], [777], [1, 1499, 700, 64, 1200]],
                                     block_q=16, chunk_kv=320, num_partitions=4, hq=8, hkv=2, d=128)):
        q, k, v, do = synth.make_tensors(prob, seed=2, backward=True)
        qd, kd, vd, dod = _dev(q, k, v, do)
        outs = []
        for flag in (0, skv.SKV_PLAN_PARTITION_QUEUES):
            plan = skv.skv_plan(prob, skv.SKV_PLAN_LPT | flag)
            ws = skv.alloc_workspace(plan)
            o, lse = skv.forward(plan, qd, kd, vd, ws, fused=False)
            grads = skv.backward(plan, qd, kd, vd, o, lse, dod, ws, deterministic=True)
            assert skv.skv_status(ws) == 0
            torch.cuda.synchronize()
            outs.append([o.cpu(), lse.cpu()] + [g.cpu() for g in grads])
        for a, b in zip(*outs):
            assert torch.equal(a, b)
