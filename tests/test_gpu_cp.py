"""Context parallelism on one GPU, through the C ABI: the ranks of a
context-parallel group are run one after another in this process (no rank
waits for another, so nothing needs them to run at the same time). Each rank
runs the forward and backward of its shard plan over its own K/V rows; the
rank partials are combined with skv_lse_combine and the dQ shares with
skv_dq_combine, and the result is compared with the fp64 oracle of the
unsplit attention (forward max-abs 2e-2 and LSE 1e-3; gradients relative
Frobenius 1e-2). The class SplitKVContextParallel is run on a one-rank NCCL
group. The exchange between ranks is covered on CPU by tests/test_cp_gloo.py."""
import os
import socket

import numpy as np
import pytest
import torch

from split_kv_block_b200 import cp, skv, synth
from test_gpu_parity import check_backward, check_forward

pytestmark = pytest.mark.gpu


def _ranks(prob, q, k, v, do, policy=skv.SKV_PLAN_LPT, fused=False):
    """Every rank's forward, then the combine; every rank's backward with the
    combined O/LSE, then the dQ sum; dK/dV scattered back to the full layout
    (rows of other ranks stay NaN until their owner writes them)."""
    R = prob.num_partitions
    qd, dod = q.cuda(), do.cuda()
    plans, shards = [], []
    o_parts, l_parts = [], []
    for r in range(R):
        plan = skv.skv_plan_shard(prob, r, policy)
        ks, vs = cp.shard_kv(plan, k.cuda()), cp.shard_kv(plan, v.cuda())
        ws = skv.alloc_workspace(plan)
        o_r, l_r = skv.forward(plan, qd, ks, vs, ws, fused=fused)
        assert skv.skv_status(ws) == 0
        plans.append(plan)
        shards.append((ks, vs, ws))
        o_parts.append(o_r)
        l_parts.append(l_r)
    o = torch.empty_like(o_parts[0])
    lse = torch.empty_like(l_parts[0])
    skv.skv_lse_combine(torch.stack(o_parts), torch.stack(l_parts), o, lse)
    dq_parts = []
    dk = torch.full(k.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    dv = torch.full(v.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    for r in range(R):
        ks, vs, ws = shards[r]
        dq_r = torch.empty(q.shape, dtype=torch.float32, device="cuda")
        dk_r = torch.full_like(ks, float("nan"))
        dv_r = torch.full_like(vs, float("nan"))
        skv.skv_attn_bwd_partial(plans[r], qd, ks, vs, o, lse, dod, dq_r, dk_r, dv_r, ws)
        assert skv.skv_status(ws) == 0
        dq_parts.append(dq_r)
        for g, kb, ke, row in cp.shard_rows(plans[r]):
            dk[kb:ke, g] = dk_r[row:row + ke - kb, 0]
            dv[kb:ke, g] = dv_r[row:row + ke - kb, 0]
    dq = torch.empty(q.shape, dtype=torch.bfloat16, device="cuda")
    skv.skv_dq_combine(torch.stack(dq_parts), dq)
    torch.cuda.synchronize()
    return o.cpu(), lse.cpu(), (dq.cpu(), dk.cpu(), dv.cpu())


def _check(prob, seed, groups=None, policy=skv.SKV_PLAN_LPT, fused=False):
    q, k, v, do = synth.make_tensors(prob, seed=seed, backward=True)
    o, lse, grads = _ranks(prob, q, k, v, do, policy, fused)
    assert not torch.isnan(grads[1]).any() and not torch.isnan(grads[2]).any(), "a K/V row no rank wrote"
    check_forward(prob, q, k, v, o, lse, groups)
    check_backward(prob, q, k, v, do, grads, groups)


def test_shards_of_ragged_problems_head_dim_64_and_128():
    _check(synth.small_problem([1001, 777, 1500], [[1000, 3, 555], [777], [1, 1499, 700, 64, 1200]], block_q=16,
                               chunk_kv=320, sub_chunks=2, num_partitions=3, hq=8, hkv=2, d=128), 1)
    _check(synth.small_problem([400, 333, 128], [[390, 7], [], [128, 5]], block_q=16, chunk_kv=128,
                               num_partitions=4, hq=8, hkv=2, d=64), 2, policy=skv.SKV_PLAN_STATIC)


def test_shards_with_the_merge_in_the_forward_tail():
    """A rank may own no key of some query tiles; the fused forward then runs
    the merge as its own launch for those rows (O = 0, LSE = -inf)."""
    _check(synth.small_problem([900, 600], [[899, 3, 450], [600, 40]], block_q=16, chunk_kv=128, num_partitions=5,
                               hq=8, hkv=2, d=128), 3, fused=True)


def test_shards_of_the_32k_workload():
    """ctx32k at full size with its 16 partitions as 16 ranks (oracle on two kv-head groups)."""
    _check(synth.make_problem(synth.WORKLOADS["ctx32k"], seed=0), 0, groups=(0, 3))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_context_parallel_class_on_a_one_rank_nccl_group():
    """SplitKVContextParallel end to end over NCCL (world size 1: the
    collectives run, the combine and dQ sum see one rank)."""
    import torch.distributed as dist
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ["MASTER_PORT"] = str(_free_port())
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        prob = synth.small_problem([1001, 777], [[1000, 3, 555], [777, 1]], block_q=16, chunk_kv=256,
                                   num_partitions=1, hq=8, hkv=2, d=128)
        q, k, v, do = synth.make_tensors(prob, seed=5, backward=True)
        layer = cp.SplitKVContextParallel(prob)
        ks, vs = cp.shard_kv(layer.plan, k.cuda()), cp.shard_kv(layer.plan, v.cuda())
        o, lse = layer.forward(q.cuda(), ks, vs)
        dq, dk_s, dv_s = layer.backward(q.cuda(), ks, vs, o, lse, do.cuda())
        torch.cuda.synchronize()
        dk = torch.zeros(k.shape, dtype=torch.bfloat16)
        dv = torch.zeros(v.shape, dtype=torch.bfloat16)
        for g, kb, ke, row in cp.shard_rows(layer.plan):
            dk[kb:ke, g] = dk_s[row:row + ke - kb, 0].cpu()
            dv[kb:ke, g] = dv_s[row:row + ke - kb, 0].cpu()
        check_forward(prob, q, k, v, o.cpu(), lse.cpu())
        check_backward(prob, q, k, v, do, (dq.cpu(), dk, dv))
    finally:
        dist.destroy_process_group()
