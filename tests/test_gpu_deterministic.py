"""skv_attn_bwd_deterministic through the C ABI: dQ summed over key tiles in
ascending key order (turn counters per query tile, kv head and warp), so two
runs give the same bits; dK/dV are the ones of skv_attn_bwd bit for bit (each
key's gradient is written by the one unit that owns it); all three within
the gradient tolerance of the fp64 oracle."""
import numpy as np
import pytest
import torch

from split_kv_block_b200 import skv, synth
from test_gpu_parity import _dev, check_backward

pytestmark = pytest.mark.gpu


def _bits(t):
    return t.view(torch.int16).cpu()


def _runs(prob, seed, n=2, policy=skv.SKV_PLAN_LPT):
    q, k, v, do = synth.make_tensors(prob, seed=seed, backward=True)
    plan = skv.skv_plan(prob, policy)
    qd, kd, vd, dod = _dev(q, k, v, do)
    ws = skv.alloc_workspace(plan)
    o, lse = skv.forward(plan, qd, kd, vd, ws)
    det = []
    for _ in range(n):
        det.append(skv.backward(plan, qd, kd, vd, o, lse, dod, ws, deterministic=True))
        assert skv.skv_status(ws) == 0
    fast = skv.backward(plan, qd, kd, vd, o, lse, dod, ws)
    assert skv.skv_status(ws) == 0
    torch.cuda.synchronize()
    return (q, k, v, do), det, fast


def _check(prob, seed, groups=None, policy=skv.SKV_PLAN_LPT):
    (q, k, v, do), det, fast = _runs(prob, seed, policy=policy)
    for dq, dk, dv in det[1:]:
        assert torch.equal(_bits(dq), _bits(det[0][0])), "dQ differs between deterministic runs"
        assert torch.equal(_bits(dk), _bits(det[0][1])) and torch.equal(_bits(dv), _bits(det[0][2]))
    assert torch.equal(_bits(det[0][1]), _bits(fast[1])) and torch.equal(_bits(det[0][2]), _bits(fast[2]))
    # the two dQ differ only by the order of fp32 additions
    a, b = det[0][0].double(), fast[0].double()
    assert float((a - b).norm() / b.norm().clamp_min(1e-30)) < 2e-3
    check_backward(prob, q, k, v, do, [g.cpu() for g in det[0]], groups)


def test_deterministic_tiny_and_ragged_head_dim_64():
    _check(synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0), 0)
    prob = synth.small_problem([400, 333, 128], [[390, 7], [], [128, 5]], block_q=16, chunk_kv=128,
                               num_partitions=3, hq=8, hkv=2, d=64)
    _check(prob, 1, policy=skv.SKV_PLAN_STATIC)


def test_deterministic_ragged_head_dim_128():
    rng = np.random.default_rng(77)
    for i in range(4):
        prob = synth.random_small_problem(rng, max_len=900, max_anchors=7, d=128,
                                          heads=((4, 1), (8, 2), (16, 2), (2, 2)))
        _check(prob, i)


def test_deterministic_ctx32k_full_size():
    """The 32K workload: many units per query tile, so the turn order is
    exercised under full concurrency; oracle on two kv-head groups."""
    _check(synth.make_problem(synth.WORKLOADS["ctx32k"], seed=0), 0, groups=(1, 6))
