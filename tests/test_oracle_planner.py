"""Pins of the planner oracle: brute-force mask counts, brute-force optimal
makespans with Graham's LPT bound (the 4/3 guarantee quoted in "Split-KV:
Breaking the Context Parallelism Bottleneck ...", section "LPT Scheduling"),
a textbook LPT instance, closed-form totals and hand-computed loads."""
import itertools
import json
import os

import numpy as np
import pytest

from oracle import planner as PL
from split_kv_block_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _mask_count(prob, b, lo, hi):
    """Brute force: build the explicit boolean mask of sample b (query token x
    key) and count True entries in keys [lo, hi), times the group size."""
    S = prob.block_q
    k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
    j0, j1 = int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])
    a_tok = np.repeat(prob.anchors[j0:j1], S)
    mask = np.arange(k1 - k0)[None, :] < a_tok[:, None]
    if prob.key_block_mask is not None:
        rows = np.repeat(prob.key_block_mask[j0:j1], S, axis=0).astype(bool)
        mask = mask & rows[:, np.arange(k1 - k0) // 128]
    G = prob.num_q_heads // prob.num_kv_heads
    return G * int(mask[:, lo - k0:hi - k0].sum())


def test_item_costs_match_mask_count():
    rng = np.random.default_rng(0)
    for _ in range(30):
        prob = synth.random_small_problem(rng)
        for it in PL.lpt_items(prob):
            assert it.cost == _mask_count(prob, it.b, it.key_begin, it.key_end)


def test_items_tile_every_context_once():
    rng = np.random.default_rng(1)
    for _ in range(30):
        prob = synth.random_small_problem(rng)
        for items in (PL.lpt_items(prob), PL.static_plan(prob)[0]):
            for g in range(prob.num_kv_heads):
                cover = np.zeros(int(prob.ctx_offsets[-1]), dtype=int)
                for it in items:
                    if it.g == g:
                        assert int(prob.ctx_offsets[it.b]) <= it.key_begin < it.key_end <= int(prob.ctx_offsets[it.b + 1])
                        cover[it.key_begin:it.key_end] += 1
                assert (cover == 1).all()


def test_total_cost_closed_form():
    """Sum of item costs = Hq * block_q * sum of anchors (every unmasked pair once)."""
    rng = np.random.default_rng(2)
    for _ in range(30):
        prob = synth.random_small_problem(rng)
        tot = prob.num_q_heads * prob.block_q * int(prob.anchors.sum())
        assert sum(it.cost for it in PL.lpt_items(prob)) == tot
        assert sum(PL.static_plan(prob)[1]) == tot


def _opt_makespan(costs, P):
    best = None
    for assign in itertools.product(range(P), repeat=len(costs)):
        m = PL.makespan(costs, assign, P)
        best = m if best is None else min(best, m)
    return best


def test_lpt_graham_bound_brute_force():
    rng = np.random.default_rng(3)
    for _ in range(150):
        P = int(rng.integers(1, 5))
        n = int(rng.integers(1, 9 if P > 2 else 11))
        costs = [int(x) for x in rng.integers(0, 30, size=n)]
        part = PL.lpt_assign(costs, P)
        lpt = PL.makespan(costs, part, P)
        opt = _opt_makespan(costs, P)
        assert lpt * 3 * P <= (4 * P - 1) * opt          # LPT <= (4/3 - 1/(3P)) OPT
        assert lpt >= opt


def test_lpt_textbook_instance():
    with open(os.path.join(GOLDEN, "lpt_textbook.json")) as f:
        g = json.load(f)
    part = PL.lpt_assign(g["jobs"], g["machines"])
    assert PL.makespan(g["jobs"], part, g["machines"]) == g["lpt_makespan"]
    assert _opt_makespan(g["jobs"], g["machines"]) == g["optimal_makespan"]


def test_lpt_few_items_one_per_partition():
    costs = [5, 9, 0, 3]
    part = PL.lpt_assign(costs, 6)
    assert len(set(part)) == 4
    # biggest job on partition 0, then 1, ...
    assert part[1] == 0 and part[0] == 1 and part[3] == 2 and part[2] == 3


def test_lpt_input_order_invariant():
    rng = np.random.default_rng(4)
    for _ in range(50):
        n = int(rng.integers(1, 40))
        costs = [int(x) for x in rng.integers(0, 8, size=n)]   # many ties
        keys = list(range(n))
        P = int(rng.integers(1, 7))
        base = PL.lpt_assign(costs, P, keys)
        perm = rng.permutation(n)
        shuffled = PL.lpt_assign([costs[i] for i in perm], P, [keys[i] for i in perm])
        for pos, i in enumerate(perm):
            assert shuffled[pos] == base[i]


def test_imbalance_hand_instance():
    assert PL.imbalance([3, 1, 2, 2]) == pytest.approx(0.5)
    assert PL.imbalance([4, 4]) == 0.0
    assert PL.imbalance([0, 0, 0]) == 0.0
    assert PL.imbalance([6, 0, 0]) == pytest.approx(2.0)


def test_static_split_hand_instance():
    """One sample of 8 tokens, anchors {2, 8}, block_q 1, 1/1 heads, P = 2:
    partition 0 owns tokens [0,4): pairs 2 (anchor 2) + 4 (anchor 8) = 6;
    partition 1 owns [4,8): 0 + 4 = 4."""
    prob = synth.small_problem([8], [[2, 8]], block_q=1, hq=1, hkv=1, chunk_kv=3, num_partitions=2)
    assert PL.static_loads_by_tokens(prob) == [6, 4]
    items, loads = PL.static_plan(prob)
    assert loads == [6, 4]
    # chunks [0,3) [3,6) [6,8); boundary 4 cuts chunk 1 into two pieces
    assert [(it.c, it.sub, it.key_begin, it.key_end, it.partition) for it in items] == [
        (0, 0, 0, 3, 0), (1, 0, 3, 4, 0), (1, 1, 4, 6, 1), (2, 0, 6, 8, 1)]


def test_static_items_match_token_loads():
    rng = np.random.default_rng(5)
    for _ in range(30):
        prob = synth.random_small_problem(rng)
        assert PL.static_plan(prob)[1] == PL.static_loads_by_tokens(prob)


def test_lpt_plan_hand_instance():
    """Two samples, chunk 4, 1 kv head of 2 q heads, block_q 1:
    sample 0 (L=8, anchors {8}) -> chunks [0,4) cost 2*4=8, [4,8) cost 8;
    sample 1 (L=6, anchors {1, 6}) -> chunk [0,4): 2*(1+4)=10, [4,6): 2*2=4.
    LPT on 2 partitions, order 10, 8 (b0 c0), 8 (b0 c1), 4:
    10 -> p0; 8 -> p1 (load 8); 8 -> p1 (loads 10 vs 8, so p1, now 16);
    4 -> p0 (14). Loads [14, 16]."""
    prob = synth.small_problem([8, 6], [[8], [1, 6]], block_q=1, hq=2, hkv=1, chunk_kv=4, num_partitions=2)
    items, loads = PL.lpt_plan(prob)
    got = {(it.b, it.c): (it.cost, it.partition) for it in items}
    assert got == {(0, 0): (8, 1), (0, 1): (8, 1), (1, 0): (10, 0), (1, 1): (4, 0)}
    assert loads == [14, 16]


def test_golden_tiny_plan_is_current():
    """The stored plan of the 4K tiny workload (written by
    tests/golden/make_golden.py from the oracle) still matches the oracle."""
    with open(os.path.join(GOLDEN, "tiny_4k_plan.json")) as f:
        g = json.load(f)
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0)
    assert prob.anchors.tolist() == g["anchors"]
    items, loads = PL.lpt_plan(prob)
    assert [[it.b, it.c, it.g, it.sub, it.key_begin, it.key_end, it.cost, it.partition] for it in items] == g["lpt_items"]
    assert loads == g["lpt_loads"]
    assert PL.static_plan(prob)[1] == g["static_loads"]



def test_item_costs_with_a_block_mask_match_mask_count():
    rng = np.random.default_rng(9)
    for _ in range(15):
        prob = synth.random_small_problem(rng)
        lens = np.diff(prob.ctx_offsets)
        stride = int((lens.max() + 127) // 128)
        mask = (rng.random((int(prob.anchor_offsets[-1]), stride)) < 0.5).astype(np.uint8)
        prob = prob.replace(key_block_mask=mask)
        for it in PL.lpt_items(prob):
            assert it.cost == _mask_count(prob, it.b, it.key_begin, it.key_end)


def test_tile_cost_hand_instance():
    """One sample of 300 keys, anchors 100 and 260, block_q 16, 4 q-heads on
    one kv head (G = 4): a query tile holds 32 tokens, i.e. both anchors (one
    tile). Key tiles of the item [0, 300): [0,128) and [128,256) hold keys the
    anchor 260 block attends, [256,300) holds key 256..259 for it: 3 live
    blocks, 3 * 128 * 128. The item [200, 300) alone: key tiles [200,300) is
    one tile, live (anchor 260): 1 block."""
    prob = synth.small_problem([300], [[100, 260]], block_q=16, hq=4, hkv=1, d=64)
    assert PL.item_tile_cost(prob, 0, 0, 300) == 3 * 128 * 128
    assert PL.item_tile_cost(prob, 0, 200, 300) == 128 * 128
    # anchors 100 and 120 only: the keys [128, 300) are attended by nobody
    prob2 = prob.replace(anchors=np.array([100, 120]))
    assert PL.item_tile_cost(prob2, 0, 0, 300) == 128 * 128


def test_tile_cost_bounds_the_exact_cost():
    """Every attended (row, key) pair lies in a live block, so the tile cost
    is at least the exact cost, and at most 128 * 128 per key tile and query
    tile of the sample."""
    rng = np.random.default_rng(12)
    for _ in range(20):
        prob = synth.random_small_problem(rng, max_len=500)
        G = prob.num_q_heads // prob.num_kv_heads
        for it in PL.lpt_items(prob):
            tc = PL.item_tile_cost(prob, it.b, it.key_begin, it.key_end)
            assert tc >= it.cost
            n_tok = (int(prob.anchor_offsets[it.b + 1]) - int(prob.anchor_offsets[it.b])) * prob.block_q
            n_qt = -(-n_tok // (128 // G))
            n_kt = -(-(it.key_end - it.key_begin) // 128)
            assert tc <= 128 * 128 * n_qt * n_kt
