"""Context parallelism across ranks on CPU: two gloo ranks started the way
torchrun starts them (MASTER_ADDR=127.0.0.1). Each rank builds its shard plan
with the library's planner (host code), computes its partial output/LSE and
its dQ share over its own items with the fp64 oracle, and exchanges them with
the module's collectives (split_kv_block_b200.cp.gather_partials / gather_dq);
the exchanged partials, merged, must equal the single-rank oracle result
("Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion Drafter
Training", section "Split-KV's Core Mechanism": exact, query-sized
aggregation). The CUDA combine kernels are checked against the oracle in
tests/test_gpu_cp.py."""
import datetime
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem():
    from split_kv_block_b200 import synth
    return synth.small_problem([300, 170], [[290, 17, 150, 64], [170, 3]], block_q=4, chunk_kv=64, sub_chunks=2,
                               num_partitions=2, hq=8, hkv=2, d=64)


def _rank_partial(prob, q, k, v, items):
    """Oracle partial over this rank's items: per item (b, g, key range) the
    chunk partial of the heads of group g, all of them merged; rows the rank
    has no key for: O = 0, LSE = -inf."""
    from oracle import attention as A
    G = prob.num_q_heads // prob.num_kv_heads
    Nq, Hq, d = q.shape
    O = torch.zeros(Nq, Hq, d, dtype=torch.float64)
    L = torch.full((Nq, Hq), -math.inf, dtype=torch.float64)
    for g in range(prob.num_kv_heads):
        parts = []
        for (b, gg, lo, hi) in items:
            if gg != g:
                continue
            o_c, l_c = A.chunk_partial(prob, q, k, v, b, lo, hi)
            hs = slice(g * G, (g + 1) * G)
            parts.append((o_c[:, hs], l_c[:, hs]))
        if not parts:
            continue
        o_g, l_g = A.lse_merge(parts)
        live = torch.isfinite(l_g)
        O[:, g * G:(g + 1) * G] = torch.where(live[..., None], o_g, torch.zeros_like(o_g))
        L[:, g * G:(g + 1) * G] = l_g
    return O, L


def _rank_backward(prob, q, k, v, o, lse, do, items):
    """Oracle dQ share and dK/dV over this rank's items (per kv-head group)."""
    from oracle import attention as A
    G = prob.num_q_heads // prob.num_kv_heads
    dq = torch.zeros(q.shape, dtype=torch.float64)
    dk = torch.zeros(k.shape, dtype=torch.float64)
    dv = torch.zeros(v.shape, dtype=torch.float64)
    for g in range(prob.num_kv_heads):
        ranges = [(b, lo, hi) for (b, gg, lo, hi) in items if gg == g]
        if not ranges:
            continue
        gq, gk, gv = A.chunked_backward(prob, q, k, v, o, lse, do, ranges=ranges)
        dq[:, g * G:(g + 1) * G] += gq[:, g * G:(g + 1) * G]
        for (b, lo, hi) in ranges:
            dk[lo:hi, g] = gk[lo:hi, g]
            dv[lo:hi, g] = gv[lo:hi, g]
    return dq, dk, dv


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from oracle import attention as A
        from split_kv_block_b200 import cp, skv, synth
        prob = _problem()
        q, k, v, do = synth.make_tensors(prob, seed=2, backward=True)
        plan = skv.skv_plan_shard(prob, rank)
        rows = cp.shard_rows(plan)
        items = []
        for g, kb, ke, row in rows:
            b = int(np.searchsorted(prob.ctx_offsets, kb, side="right") - 1)
            items.append((b, g, kb, ke))
        o_r, l_r = _rank_partial(prob, q, k, v, items)
        o_all, l_all = cp.gather_partials(o_r, l_r)
        assert o_all.shape[0] == world and torch.equal(o_all[rank], o_r)
        O, L = A.lse_merge([(o_all[r], l_all[r]) for r in range(world)])
        dq_r, dk_r, dv_r = _rank_backward(prob, q, k, v, O, L, do, items)
        dq_all = cp.gather_dq(dq_r)
        dq = dq_all.sum(0)
        torch.save({"O": O, "L": L, "dq": dq, "dk": dk_r, "dv": dv_r, "rows": rows,
                    "kv_layout": plan.kv_layout()}, os.path.join(out_dir, f"rank{rank}.pt"))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_and_merge_equal_the_unsplit_oracle(tmp_path):
    import sys
    sys.path.insert(0, ROOT)
    from oracle import attention as A
    from split_kv_block_b200 import synth
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True, start_method="spawn")
    res = [torch.load(tmp_path / f"rank{r}.pt") for r in range(world)]
    prob = _problem()
    q, k, v, do = synth.make_tensors(prob, seed=2, backward=True)
    O_ref, L_ref = A.attention_forward(prob, q, k, v)
    gq, gk, gv = A.attention_backward(prob, q, k, v, O_ref, L_ref, do)
    for r in range(world):
        assert torch.allclose(res[r]["O"], O_ref, atol=1e-12, rtol=0)
        assert torch.allclose(res[r]["L"], L_ref, atol=1e-12, rtol=0)
        assert torch.allclose(res[r]["dq"], gq, atol=1e-11, rtol=0)
    # every (key, kv head) belongs to exactly one rank; its dK/dV there are the unsplit ones
    owner = torch.zeros(k.shape[0], k.shape[1], dtype=torch.int32)
    dk = torch.zeros_like(gk)
    dv = torch.zeros_like(gv)
    for r in range(world):
        rows_r, heads_r, shard_r = res[r]["kv_layout"]
        assert heads_r == 1 and shard_r == r
        assert rows_r == sum(ke - kb for (_, kb, ke, _) in res[r]["rows"])
        for g, kb, ke, row in res[r]["rows"]:
            owner[kb:ke, g] += 1
            dk[kb:ke, g] = res[r]["dk"][kb:ke, g]
            dv[kb:ke, g] = res[r]["dv"][kb:ke, g]
    assert torch.all(owner == 1)
    assert torch.allclose(dk, gk, atol=1e-11, rtol=0) and torch.allclose(dv, gv, atol=1e-11, rtol=0)


def test_shard_layout_of_every_rank():
    """The shard plans of all ranks: each rank's K/V rows are its items' keys
    (one kv head per row) in (b, c, g, s) order, cp.shard_kv places exactly
    those rows, and the ranks' rows together hold every (key, kv head) once."""
    import sys
    sys.path.insert(0, ROOT)
    from split_kv_block_b200 import cp, skv, synth
    prob = synth.small_problem([700, 390, 128], [[650, 129, 300], [390, 200], [128]], block_q=16, chunk_kv=128,
                               sub_chunks=2, num_partitions=3, hq=8, hkv=2, d=64)
    _, k, _, _ = synth.make_tensors(prob, seed=1, backward=False)
    seen = torch.zeros(k.shape[0], k.shape[1], dtype=torch.int32)
    for r in range(prob.num_partitions):
        plan = skv.skv_plan_shard(prob, r)
        rows, heads, shard = plan.kv_layout()
        assert heads == 1 and shard == r
        ks = cp.shard_kv(plan, k)
        assert tuple(ks.shape) == (rows, 1, k.shape[-1])
        it = plan.items()
        mine = it[it["partition"] == r]
        assert (it["kv_row"][it["partition"] != r] == -1).all()
        order = np.lexsort((mine["sub"], mine["g"], mine["c"], mine["b"]))
        row = 0
        for i in order:
            g, kb, ke = int(mine["g"][i]), int(mine["key_begin"][i]), int(mine["key_end"][i])
            assert int(mine["kv_row"][i]) == row
            assert torch.equal(ks[row:row + ke - kb, 0], k[kb:ke, g])
            seen[kb:ke, g] += 1
            row += ke - kb
        assert row == rows
    assert torch.all(seen == 1)
