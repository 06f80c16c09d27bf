"""Block-sparse masks through the C ABI: per (anchor, 128-key block) mask
bytes on top of the prefix mask ("Split-KV: Efficient Context Parallelism for
Training Diffusion Drafters", Abstract: cross-attention with a block-sparse
mask over the context). The kernels walk only the key tiles a tile attends
(forward) and the query tiles that attend a key tile (backward), and mask the
rows whose block is off. Element by element against the fp64 oracle, with the
forward tolerances (O 2e-2, LSE 1e-3) and the gradient tolerance (relative
Frobenius 1e-2)."""
import numpy as np
import pytest
import torch

from split_kv_block_b200 import cp, skv, synth
from test_gpu_parity import _case, check_backward, check_forward, run_gpu

pytestmark = pytest.mark.gpu


def _random_mask(prob, rng, density):
    lens = np.diff(prob.ctx_offsets)
    stride = int((lens.max() + 127) // 128)
    return prob.replace(key_block_mask=(rng.random((int(prob.anchor_offsets[-1]), stride)) < density)
                        .astype(np.uint8))


@pytest.mark.parametrize("d", [64, 128])
def test_random_masks_on_ragged_problems(d):
    """Random masks of several densities (including rows left with no key),
    ragged samples and tiles, LPT plans with sub-chunks; forward through the
    merge kernel and through the merge in the forward's tail."""
    rng = np.random.default_rng(500 + d)
    for i in range(5):
        prob = synth.random_small_problem(rng, max_len=1400, max_anchors=7, d=d,
                                          heads=((4, 1), (8, 2), (16, 2), (2, 2)))
        chunk = int(rng.choice([128, 256, 384]))
        prob = prob.replace(chunk_kv=chunk, sub_chunks=1 if chunk != 256 else 2)
        prob = _random_mask(prob, rng, density=(0.15, 0.4, 0.7, 1.0, 0.3)[i])
        _case(prob, seed=i, fused=i % 2 == 0)


def test_mask_workload_full_size():
    """ctx32k shapes under the sink + window + random-block mask, full size;
    oracle on two kv-head groups."""
    prob = synth.make_problem(synth.WORKLOADS["ctx32k_sparse"], seed=0)
    _case(prob, groups=(2, 5))


def test_mask_with_bf16_partials_deterministic_backward_and_shards():
    """The mask together with the other options: bf16 partial outputs, the
    deterministic backward (two runs, identical dQ bits), and context-parallel
    shards combined with skv_lse_combine."""
    rng = np.random.default_rng(9)
    prob = synth.small_problem([1400, 900], [[1300, 5, 700, 256], [899, 200, 640]], block_q=16, chunk_kv=256,
                               sub_chunks=2, num_partitions=3, hq=8, hkv=2, d=128)
    prob = _random_mask(prob, rng, 0.5)
    q, k, v, do = synth.make_tensors(prob, seed=4, backward=True)
    o, lse, _, _ = run_gpu(prob, q, k, v, None, skv.SKV_PLAN_LPT | skv.SKV_PLAN_PARTIALS_BF16)
    check_forward(prob, q, k, v, o, lse)
    plan = skv.skv_plan(prob)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    ws = skv.alloc_workspace(plan)
    o, lse = skv.forward(plan, qd, kd, vd, ws)
    g1 = skv.backward(plan, qd, kd, vd, o, lse, dod, ws, deterministic=True)
    g2 = skv.backward(plan, qd, kd, vd, o, lse, dod, ws, deterministic=True)
    assert skv.skv_status(ws) == 0
    assert torch.equal(g1[0].view(torch.int16), g2[0].view(torch.int16))
    check_backward(prob, q, k, v, do, [g.cpu() for g in g1])
    # shards: every rank's partial over its own rows, then the exact combine
    parts = []
    for r in range(prob.num_partitions):
        sp = skv.skv_plan_shard(prob, r)
        ks, vs = cp.shard_kv(sp, kd), cp.shard_kv(sp, vd)
        parts.append(skv.forward(sp, qd, ks, vs, skv.alloc_workspace(sp), fused=False))
    oc, lc = torch.empty_like(o), torch.empty_like(lse)
    skv.skv_lse_combine(torch.stack([x[0] for x in parts]), torch.stack([x[1] for x in parts]), oc, lc)
    torch.cuda.synchronize()
    check_forward(prob, q, k, v, oc.cpu(), lc.cpu())
