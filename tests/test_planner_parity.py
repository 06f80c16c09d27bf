"""The C++ planner (skv_plan through the C ABI) against the planner oracle:
items, realized costs, partitions and partition loads must be bit-exact
("Split-KV: Breaking the Context Parallelism Bottleneck ...", section "LPT
Scheduling"). Host-only: runs without a GPU."""
import ctypes

import numpy as np
import pytest

from oracle import planner as PL
from split_kv_block_b200 import skv, synth


def _compare(prob, policy):
    plan = skv.skv_plan(prob, policy)
    got = plan.items()
    if policy == skv.SKV_PLAN_LPT:
        ref, loads = PL.lpt_plan(prob)
    elif policy == skv.SKV_PLAN_LPT_TILES:
        ref, loads = PL.lpt_plan(prob, cost="tiles")
    else:
        ref, loads = PL.static_plan(prob)
    assert len(got) == len(ref)
    mine = [(int(r["b"]), int(r["c"]), int(r["g"]), int(r["sub"]), int(r["key_begin"]), int(r["key_end"]),
             int(r["cost"]), int(r["partition"])) for r in got]
    theirs = [(it.b, it.c, it.g, it.sub, it.key_begin, it.key_end, it.cost, it.partition) for it in ref]
    assert mine == theirs
    assert plan.partition_load.tolist() == loads
    st = plan.stats()
    assert st["total_cost"] == sum(loads)
    assert st["imbalance"] == pytest.approx(PL.imbalance(loads), abs=1e-12)
    return plan


@pytest.mark.parametrize("name", sorted(synth.WORKLOADS))
@pytest.mark.parametrize("policy", [skv.SKV_PLAN_LPT, skv.SKV_PLAN_STATIC])
def test_workloads_bit_exact(name, policy):
    for seed in range(3):
        prob = synth.make_problem(synth.WORKLOADS[name], seed=seed)
        _compare(prob, policy)


def test_ctx128k_subchunks_bit_exact():
    prob = synth.make_problem(synth.WORKLOADS["ctx128k"], seed=0, sub_chunks=4)
    _compare(prob, skv.SKV_PLAN_LPT)


def test_random_small_problems_bit_exact():
    rng = np.random.default_rng(2024)
    for i in range(1000):
        prob = synth.random_small_problem(rng)
        _compare(prob, skv.SKV_PLAN_LPT if i % 2 == 0 else skv.SKV_PLAN_STATIC)


def test_more_partitions_than_items():
    prob = synth.small_problem([100], [[50]], chunk_kv=64, num_partitions=9, hq=2, hkv=1)
    plan = _compare(prob, skv.SKV_PLAN_LPT)
    parts = sorted(int(x) for x in plan.items()["partition"])
    assert parts == [0, 1]


def test_single_partition():
    prob = synth.small_problem([300, 70], [[300, 2], [5]], chunk_kv=64, num_partitions=1)
    plan = _compare(prob, skv.SKV_PLAN_LPT)
    assert plan.stats()["imbalance"] == 0.0


def test_zero_anchor_sample():
    prob = synth.small_problem([200, 90], [[150], []], chunk_kv=64, num_partitions=3)
    _compare(prob, skv.SKV_PLAN_LPT)
    _compare(prob, skv.SKV_PLAN_STATIC)


def _status(prob, policy=skv.SKV_PLAN_LPT):
    try:
        skv.skv_plan_size(prob, policy)
        return 0
    except skv.SkvError as e:
        return e.code


def test_invalid_arguments_rejected():
    ok = synth.small_problem([100], [[50]])
    assert _status(ok) == 0
    assert _status(ok.replace(anchors=np.array([0]))) == 1            # a < 1
    assert _status(ok.replace(anchors=np.array([101]))) == 1          # a > L
    assert _status(ok.replace(num_kv_heads=3)) == 1                   # Hq % Hkv
    assert _status(ok.replace(chunk_kv=100, sub_chunks=3)) == 1       # C % sub
    assert _status(ok.replace(num_partitions=0)) == 1
    assert _status(ok.replace(block_q=0)) == 1
    assert _status(ok, policy=7) == 1
    assert _status(ok.replace(ctx_offsets=np.array([0, 0]), anchors=np.zeros(0, np.int64),
                              anchor_offsets=np.array([0, 0], np.int32))) == 1   # empty sample
    assert _status(ok.replace(head_dim=96)) == 3                      # unsupported d
    assert _status(ok.replace(num_q_heads=24, num_kv_heads=1)) == 3   # group of 24 rows does not tile 128


def test_plan_buffer_too_small():
    prob = synth.small_problem([100], [[50]])
    sizes = skv.skv_plan_size(prob)
    small = np.empty(sizes.plan_bytes - 1, dtype=np.uint8)
    with pytest.raises(skv.SkvError) as e:
        skv.skv_plan(prob, sizes=skv.PlanSizes(sizes.n_items, sizes.plan_bytes - 1, 0, 0), buf=small)
    assert e.value.code == 2


def test_plan_is_deterministic():
    prob = synth.make_problem(synth.WORKLOADS["batch8_logu"], seed=1)
    a = skv.skv_plan(prob)
    b = skv.skv_plan(prob)
    assert a.buf.tobytes() == b.buf.tobytes()


def test_library_exports_every_declared_symbol():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "skv.h")).read()
    declared = set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(skv_[a-z_0-9]+)\s*\(", hdr, re.M))
    assert declared == set(skv.EXPORTS)
    L = skv.lib()
    for name in declared:
        assert hasattr(L, name), name


def _expected_unit_counts(prob, items):
    """Forward / backward work units per partition, counted from the items and
    the anchors alone: a forward unit is an (item, 128-row query tile) whose
    tile reaches past the item's first key; a backward unit is a 128-key tile
    of an item below the sample's largest anchor."""
    P = prob.num_partitions
    G = prob.num_q_heads // prob.num_kv_heads
    tok_per_tile = 128 // G
    fwd, bwd = np.zeros(P, np.int64), np.zeros(P, np.int64)
    tiles = {}
    for b in range(prob.num_samples):
        j0, j1 = int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])
        a = [int(x) for x in prob.anchors[j0:j1]]
        ntok = (j1 - j0) * prob.block_q
        base = int(prob.ctx_offsets[b])
        tiles[b] = [base + max(a[t // prob.block_q] for t in range(t0, min(t0 + tok_per_tile, ntok)))
                    for t0 in range(0, ntok, tok_per_tile)]
    for it in items:
        b, kb, ke, p = int(it["b"]), int(it["key_begin"]), int(it["key_end"]), int(it["partition"])
        fwd[p] += sum(1 for kmax in tiles[b] if min(ke, kmax) > kb)
        kmax_b = max(tiles[b]) if tiles[b] else int(prob.ctx_offsets[b])
        bwd[p] += len(range(kb, min(ke, kmax_b), 128))
    return fwd, bwd


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_unit_partitions_match_item_partitions(seed):
    rng = np.random.default_rng(500 + seed)
    prob = synth.random_small_problem(rng, max_len=3000, max_anchors=9, d=128, heads=((8, 2), (16, 4), (4, 1)))
    P = prob.num_partitions
    for flag in (0, skv.SKV_PLAN_PARTITION_QUEUES):
        plan = skv.skv_plan(prob, skv.SKV_PLAN_LPT | flag)
        fp, bp = plan.unit_partitions()
        st = plan.stats()
        assert len(fp) == st["n_fwd_units"] and len(bp) == st["n_bwd_units"]
        assert np.all((fp >= 0) & (fp < P)) and np.all((bp >= 0) & (bp < P))
        if flag:  # one work queue per partition: the work lists are grouped by partition
            assert np.all(np.diff(fp) >= 0) and np.all(np.diff(bp) >= 0)
        ef, eb = _expected_unit_counts(prob, plan.items())
        assert np.bincount(fp, minlength=P).tolist() == ef.tolist()
        assert np.bincount(bp, minlength=P).tolist() == eb.tolist()


def test_unit_partitions_of_the_32k_workload():
    prob = synth.make_problem(synth.WORKLOADS["ctx32k"], seed=0)
    plan = skv.skv_plan(prob)
    fp, bp = plan.unit_partitions()
    ef, eb = _expected_unit_counts(prob, plan.items())
    P = prob.num_partitions
    assert np.bincount(fp, minlength=P).tolist() == ef.tolist()
    assert np.bincount(bp, minlength=P).tolist() == eb.tolist()


def test_plans_do_not_depend_on_earlier_calls():
    """The planner reuses its working memory between calls on a thread: a plan
    must come out byte-identical whatever was planned before it (larger,
    smaller, other policy)."""
    rng = np.random.default_rng(77)
    big = synth.make_problem(synth.WORKLOADS["ctx128k"], seed=1, sub_chunks=4)
    small = synth.random_small_problem(rng, max_len=900, max_anchors=5, d=64, heads=((4, 1),))
    other = synth.make_problem(synth.WORKLOADS["ctx32k"], seed=2)
    ref = {name: {pol: skv.skv_plan(p, pol).buf.tobytes() for pol in (skv.SKV_PLAN_LPT, skv.SKV_PLAN_STATIC)}
           for name, p in (("big", big), ("small", small), ("other", other))}
    order = [("small", small), ("big", big), ("other", other), ("small", small), ("big", big), ("small", small)]
    for name, p in order:
        for pol in (skv.SKV_PLAN_STATIC, skv.SKV_PLAN_LPT):
            assert skv.skv_plan(p, pol).buf.tobytes() == ref[name][pol], (name, pol)


def test_plan_bytes_do_not_depend_on_the_buffer_contents():
    """skv_plan writes every byte of the plan, the alignment gaps between its
    arrays included: a buffer full of 0xFF and a zeroed one give the same bytes
    (plain, block-masked, shard and deterministic-backward arrays)."""
    rng = np.random.default_rng(5)
    probs = [synth.make_problem(synth.WORKLOADS["ctx32k"], seed=0),
             synth.make_problem(synth.WORKLOADS["ctx32k_sparse"], seed=0),
             synth.make_problem(synth.WORKLOADS["batch8_logu"], seed=3),
             synth.random_small_problem(rng, max_len=900, max_anchors=5, d=64, heads=((4, 1),))]
    for p in probs:
        for pol in (skv.SKV_PLAN_LPT, skv.SKV_PLAN_STATIC, skv.SKV_PLAN_LPT | skv.SKV_PLAN_PARTITION_QUEUES):
            try:
                sizes = skv.skv_plan_size(p, pol)
            except skv.SkvError:
                continue
            a = np.zeros(sizes.plan_bytes, np.uint8)
            b = np.full(sizes.plan_bytes, 0xFF, np.uint8)
            skv.skv_plan(p, pol, sizes=sizes, buf=a)
            skv.skv_plan(p, pol, sizes=sizes, buf=b)
            assert a.tobytes() == b.tobytes(), pol
        for part in range(min(3, p.num_partitions)):
            sizes = skv.skv_plan_shard_size(p, part)
            bufs = []
            for fill in (0x00, 0xFF):
                buf = np.full(sizes.plan_bytes, fill, np.uint8)
                loads = np.zeros(p.num_partitions, np.int64)
                rc = skv.lib().skv_plan_shard(skv._ProblemArgs(p).ref(), skv.SKV_PLAN_LPT, part,
                                              ctypes.c_void_p(buf.ctypes.data), buf.nbytes,
                                              ctypes.c_void_p(loads.ctypes.data))
                assert rc == 0
                bufs.append(buf.tobytes())
            assert bufs[0] == bufs[1], part


def _fake_dev(n=8):
    """Non-NULL, 256-byte aligned addresses that no call may dereference: every
    call below is refused on the host before it enqueues anything."""
    return [ctypes.c_void_p(0x100000 + 0x1000 * i) for i in range(n)]


def test_plan_for_another_problem_is_refused_before_any_launch():
    """A plan is bound to the problem it was made for (the library stores a
    hash of the problem in it). Every call that runs kernels takes the
    problem too and returns SKV_EPLAN, on the host, when they differ: other
    anchors with the same sizes, more anchors (a larger Nq), a longer context,
    another head count. With the matching problem the same calls pass the
    check (here they would then need a GPU, so only refusals run on CPU)."""
    L = skv.lib()
    base = synth.small_problem([700, 300], [[5, 600, 41], [300]], block_q=16, chunk_kv=256, hq=8, hkv=2, d=128)
    plan = skv.skv_plan(base)
    others = [base.replace(anchors=np.array([5, 601, 41, 300], dtype=np.int64)),
              synth.small_problem([700, 300], [[5, 600, 41, 7], [300]], block_q=16, chunk_kv=256, hq=8, hkv=2,
                                  d=128),
              synth.small_problem([701, 300], [[5, 600, 41], [300]], block_q=16, chunk_kv=256, hq=8, hkv=2, d=128),
              base.replace(num_q_heads=16),
              base.replace(num_partitions=5)]
    f = _fake_dev()
    for other in others:
        pr = skv._ProblemArgs(other).ref()
        assert L.skv_attn_fwd(plan.ptr, pr, f[0], f[1], f[2], f[3], 1 << 30, None) == 5
        assert L.skv_attn_fwd_merged(plan.ptr, pr, f[0], f[1], f[2], f[4], f[5], f[3], 1 << 30, None) == 5
        assert L.skv_lse_merge(plan.ptr, pr, f[3], f[4], f[5], None) == 5
        assert L.skv_attn_bwd(plan.ptr, pr, *f[:7], f[7], f[0], f[1], 1 << 30, None) == 5
        assert L.skv_attn_bwd_deterministic(plan.ptr, pr, *f[:7], f[7], f[0], f[1], 1 << 30, None) == 5
        assert L.skv_attn_fwd_noalloc(plan.ptr, pr, f[0], f[1], f[2], f[3], f[4], None) == 5
    # NULL problem: invalid argument; a buffer that is not a plan: SKV_EPLAN
    assert L.skv_attn_fwd(plan.ptr, None, f[0], f[1], f[2], f[3], 1 << 30, None) == 1
    junk = np.zeros(plan.buf.nbytes, dtype=np.uint8)
    assert L.skv_attn_fwd(ctypes.c_void_p(junk.ctypes.data), plan.prob_ref, f[0], f[1], f[2], f[3], 1 << 30,
                          None) == 5


def test_bf16_partials_flag_changes_only_the_partial_workspace():
    """SKV_PLAN_PARTIALS_BF16 keeps items, placement and work lists; the
    forward workspace shrinks by half the partial outputs' bytes; unknown
    policy bits are refused."""
    prob = synth.make_problem(synth.WORKLOADS["ctx32k"], seed=0)
    a = skv.skv_plan(prob, skv.SKV_PLAN_LPT)
    b = skv.skv_plan(prob, skv.SKV_PLAN_LPT | skv.SKV_PLAN_PARTIALS_BF16)
    assert np.array_equal(a.items(), b.items())
    assert a.stats() == b.stats()
    n_fwd = a.stats()["n_fwd_units"]
    saved = a.sizes.ws_fwd_bytes - b.sizes.ws_fwd_bytes
    assert n_fwd * 128 * 128 * 2 - 256 <= saved <= n_fwd * 128 * 128 * 2 + 256
    assert a.sizes.ws_bwd_bytes == b.sizes.ws_bwd_bytes
    st = skv.skv_plan(prob, skv.SKV_PLAN_STATIC | skv.SKV_PLAN_PARTIALS_BF16)
    assert np.array_equal(st.items(), skv.skv_plan(prob, skv.SKV_PLAN_STATIC).items())
    for bad in (3, 0x400, 0x101 | 0x800):
        with pytest.raises(skv.SkvError):
            skv.skv_plan_size(prob, bad)


def _masked_problem(rng, density=0.5):
    prob = synth.random_small_problem(rng, max_len=1500, max_anchors=6)
    chunk = int(rng.choice([128, 256, 512]))
    sub = int(rng.choice([s for s in (1, 2, 4) if (chunk // s) % 128 == 0]))
    lens = np.diff(prob.ctx_offsets)
    stride = int((lens.max() + 127) // 128) + int(rng.integers(0, 3))
    mask = (rng.random((int(prob.anchor_offsets[-1]), stride)) < density).astype(np.uint8)
    return prob.replace(chunk_kv=chunk, sub_chunks=sub, key_block_mask=mask)


def test_block_mask_plans_bit_exact():
    """Items, realized costs under a block-sparse mask, LPT partitions and
    loads: bit-exact to the oracle planner on random masked problems, for the
    LPT plan and for the static split (whose pieces cut blocks: partial blocks
    counted key by key)."""
    rng = np.random.default_rng(31)
    for i in range(200):
        prob = _masked_problem(rng)
        _compare(prob, skv.SKV_PLAN_LPT)
        if i % 4 == 0:
            _compare(prob, skv.SKV_PLAN_STATIC)
    for i in range(20):  # chunks that are not a multiple of 128 keys
        prob = _masked_problem(rng).replace(chunk_kv=int(rng.choice([100, 320])), sub_chunks=1)
        _compare(prob, skv.SKV_PLAN_LPT)
    w = synth.WORKLOADS["ctx32k"]
    prob = synth.make_problem(w, seed=0)
    prob = prob.replace(key_block_mask=synth.block_mask_sink_window_random(prob, seed=0))
    _compare(prob, skv.SKV_PLAN_LPT)


def test_block_mask_refusals():
    """Plans whose items do not start on 128-key blocks (the static split's
    pieces, chunks that are not a multiple of 128 keys) are made for their
    costs and loads, but every kernel call refuses them on the host
    (SKV_EUNSUPPORTED); a mask row shorter than a sample's block count is
    refused by the planner."""
    rng = np.random.default_rng(4)
    # one 1000-key sample on 3 partitions: the static split cuts at keys 333 and 666
    prob = synth.small_problem([1000], [[999, 400, 100]], block_q=16, chunk_kv=256, num_partitions=3, hq=8, hkv=2,
                               d=128)
    prob = prob.replace(key_block_mask=(rng.random((3, 8)) < 0.6).astype(np.uint8))
    f = _fake_dev()
    L = skv.lib()
    for plan in (skv.skv_plan(prob, skv.SKV_PLAN_STATIC), skv.skv_plan(prob.replace(chunk_kv=320, sub_chunks=1))):
        pr = plan.prob_ref
        assert L.skv_attn_fwd(plan.ptr, pr, f[0], f[1], f[2], f[3], 1 << 30, None) == 3
        assert L.skv_attn_fwd_merged(plan.ptr, pr, f[0], f[1], f[2], f[4], f[5], f[3], 1 << 30, None) == 3
        assert L.skv_lse_merge(plan.ptr, pr, f[3], f[4], f[5], None) == 3
        assert L.skv_attn_bwd(plan.ptr, pr, *f[:7], f[7], f[0], f[1], 1 << 30, None) == 3
        assert L.skv_attn_fwd_noalloc(plan.ptr, pr, f[0], f[1], f[2], f[3], f[4], None) == 3
    lens = np.diff(prob.ctx_offsets)
    short = prob.key_block_mask[:, :int((lens.max() + 127) // 128) - 1]
    with pytest.raises(skv.SkvError) as e:
        skv.skv_plan(prob.replace(key_block_mask=np.ascontiguousarray(short)))
    assert e.value.code == 1


def test_block_mask_changes_the_fingerprint():
    """A plan made for one mask is refused with another mask of the same shape."""
    rng = np.random.default_rng(6)
    prob = _masked_problem(rng)
    plan = skv.skv_plan(prob)
    other = prob.key_block_mask.copy()
    other[0, 0] ^= 1
    f = _fake_dev()
    pr = skv._ProblemArgs(prob.replace(key_block_mask=other)).ref()
    assert skv.lib().skv_attn_fwd(plan.ptr, pr, f[0], f[1], f[2], f[3], 1 << 30, None) == 5



def test_tile_cost_plans_bit_exact():
    """SKV_PLAN_LPT_TILES (LPT on the executed-tile cost): items, costs,
    partitions and loads bit-exact to the oracle, on the tiny workload and on
    random problems with and without block masks."""
    _compare(synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0), skv.SKV_PLAN_LPT_TILES)
    rng = np.random.default_rng(77)
    for i in range(60):
        prob = synth.random_small_problem(rng, max_len=600)
        if i % 3 == 0:
            prob = _masked_problem(rng)
            prob = prob.replace(ctx_offsets=prob.ctx_offsets)  # aligned chunks from _masked_problem
        _compare(prob, skv.SKV_PLAN_LPT_TILES)


def test_tile_cost_at_least_the_exact_cost_on_the_workloads():
    """On the benchmark workloads the executed tile work exceeds the attended
    work by the tile rounding (and the two anchors that share a query tile)."""
    for name in ("ctx32k", "ctx128k", "batch8_logu"):
        prob = synth.make_problem(synth.WORKLOADS[name], seed=0)
        exact = skv.skv_plan(prob).stats()["total_cost"]
        tiles = skv.skv_plan(prob, skv.SKV_PLAN_LPT_TILES).stats()["total_cost"]
        assert exact <= tiles <= 1.2 * exact


def test_partition_queues_flag_changes_only_the_queues():
    """SKV_PLAN_PARTITION_QUEUES keeps the items, costs, partitions, loads
    and the K/V layout; unknown bits stay refused."""
    for name in ("ctx32k", "batch8_logu"):
        prob = synth.make_problem(synth.WORKLOADS[name], seed=0)
        for policy in (skv.SKV_PLAN_LPT, skv.SKV_PLAN_STATIC):
            a = skv.skv_plan(prob, policy)
            b = skv.skv_plan(prob, policy | skv.SKV_PLAN_PARTITION_QUEUES)
            assert np.array_equal(a.items(), b.items())
            assert np.array_equal(a.partition_load, b.partition_load)
            assert a.stats() == b.stats()
            # the workspace holds the plan's device lists: only the queue offsets grow (3 x P int32)
            for x, y in ((b.sizes.ws_fwd_bytes, a.sizes.ws_fwd_bytes), (b.sizes.ws_bwd_bytes, a.sizes.ws_bwd_bytes)):
                assert 0 <= x - y <= 3 * 4 * prob.num_partitions + 3 * 256
            assert a.kv_layout()[0] == b.kv_layout()[0]
    with pytest.raises(skv.SkvError):
        skv.skv_plan_size(prob, 0x400 | skv.SKV_PLAN_PARTITION_QUEUES)
