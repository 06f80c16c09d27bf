"""CPU oracle: split-KV work items, realized cost, LPT and the static split.

Test infrastructure only (see oracle/__init__.py).

[Article] "LPT Scheduling": with the global query view, Split-KV weighs each
context KV block by the attention cost it actually incurs and places blocks
with longest-processing-time-first: jobs sorted longest first, each given to
the currently least-loaded machine; classic LPT carries a 4/3 approximation
guarantee. The traditional practice it replaces splits the context roughly
by token count. [Abstract]: LPT "balances context key/value chunks by their
realized attention cost" and reaches < 1% imbalance.

Readings (the pages give no formula):
  * item = (sample b, chunk c, kv-head g, key sub-chunk s); chunk c of a
    sample of length L is [cC, min((c+1)C, L)); sub-chunk s is
    [cC + s*C/sub, min(cC + (s+1)*C/sub, chunk end)), empty ones dropped;
  * realized cost of an item = number of unmasked (query token, key) pairs
    in its key range, times the q-heads of its group:
        G * sum_j block_q * |[lo, hi) intersect [0, a_j)|   (exact, int);
  * LPT order: cost descending, then (b, c, g, s) ascending; each item goes
    to the partition with the smallest (load, index); zero-cost items take
    part like the others;
  * static split: partition p owns tokens [floor(p T / P), floor((p+1) T / P))
    of the packed context stream (T = sum of L_b) with all heads; its pieces
    are cut at chunk boundaries and become items (b, c, g, s = piece index
    within the chunk);
  * imbalance = max_p load_p / mean_p load_p - 1, mean over all P partitions
    (0 when every load is 0).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List


@dataclass(frozen=True)
class Item:
    b: int
    c: int
    g: int
    sub: int
    key_begin: int   # absolute index in the packed context
    key_end: int
    cost: int
    partition: int = -1


def item_cost(prob, b: int, key_begin: int, key_end: int) -> int:
    """G * sum over the sample's anchors of block_q * |[lo, hi) ∩ [0, a)|,
    written as a plain loop (relative key coordinates). With a block-sparse
    mask only the keys whose 128-key block is set for the anchor count."""
    G = prob.num_q_heads // prob.num_kv_heads
    k0 = int(prob.ctx_offsets[b])
    lo, hi = key_begin - k0, key_end - k0
    mask = getattr(prob, "key_block_mask", None)
    pairs = 0
    for j in range(int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])):
        a = int(prob.anchors[j])
        if mask is None:
            pairs += prob.block_q * max(0, min(hi, a) - lo)
        else:
            for kk in range(lo, min(hi, a)):
                if mask[j][kk // 128]:
                    pairs += prob.block_q
    return G * pairs


TILE_M = 128   # query rows per tile: 128 / G consecutive tokens x the G q-heads of a kv group
TILE_N = 128   # keys per key tile


def item_tile_cost(prob, b: int, key_begin: int, key_end: int) -> int:
    """Cost calibrated to the work the kernels execute (a
    refinement of the realized cost): the query rows of sample b are cut into
    tiles of 128 / G consecutive tokens (G q-heads each, 128 rows), the item's
    keys into tiles of 128 keys from key_begin; every (query tile, key tile)
    block in which some token attends some key runs as a whole 128 x 128
    block, so the cost is 128 * 128 per such block. Plain loops."""
    G = prob.num_q_heads // prob.num_kv_heads
    tt = TILE_M // G
    S = prob.block_q
    k0 = int(prob.ctx_offsets[b])
    t_begin, t_end = int(prob.anchor_offsets[b]) * S, int(prob.anchor_offsets[b + 1]) * S
    mask = getattr(prob, "key_block_mask", None)
    blocks = 0
    for t0 in range(t_begin, t_end, tt):
        tokens = range(t0, min(t0 + tt, t_end))
        for kb in range(key_begin, key_end, TILE_N):
            ke = min(kb + TILE_N, key_end)
            live = False
            for tok in tokens:
                j = tok // S
                a = int(prob.anchors[j])
                for kk in range(kb - k0, ke - k0):
                    if kk < a and (mask is None or mask[j][kk // 128]):
                        live = True
                        break
                if live:
                    break
            blocks += live
    return TILE_M * TILE_N * blocks


def lpt_items(prob, cost: str = "exact") -> List[Item]:
    """All (b, c, g, s) items in (b, c, g, s) order, with their cost: the
    realized attention cost ("exact") or the executed tile work ("tiles")."""
    C, sub = prob.chunk_kv, prob.sub_chunks
    cost_fn = item_tile_cost if cost == "tiles" else item_cost
    cs = C // sub
    items = []
    for b in range(prob.num_samples):
        k0 = int(prob.ctx_offsets[b])
        L = int(prob.ctx_offsets[b + 1]) - k0
        for c in range((L + C - 1) // C):
            c_end = min((c + 1) * C, L)
            for g in range(prob.num_kv_heads):
                for s in range(sub):
                    lo, hi = c * C + s * cs, min(c * C + (s + 1) * cs, c_end)
                    if hi <= lo:
                        continue
                    items.append(Item(b, c, g, s, k0 + lo, k0 + hi, cost_fn(prob, b, k0 + lo, k0 + hi)))
    return items


def lpt_assign(costs: List[int], num_partitions: int, keys=None) -> List[int]:
    """Longest processing time first. `keys` breaks ties between equal costs
    (default: the job index). Returns the partition of every job."""
    n = len(costs)
    if keys is None:
        keys = list(range(n))
    order = sorted(range(n), key=lambda i: (-costs[i], keys[i]))
    load = [0] * num_partitions
    part = [-1] * n
    for i in order:
        best = 0
        for p in range(1, num_partitions):          # smallest (load, p)
            if load[p] < load[best]:
                best = p
        part[i] = best
        load[best] += costs[i]
    return part


def lpt_plan(prob, cost: str = "exact"):
    """Returns (items with partitions, partition loads)."""
    items = lpt_items(prob, cost)
    part = lpt_assign([it.cost for it in items], prob.num_partitions,
                      keys=[(it.b, it.c, it.g, it.sub) for it in items])
    out = [Item(it.b, it.c, it.g, it.sub, it.key_begin, it.key_end, it.cost, p) for it, p in zip(items, part)]
    return out, partition_loads(out, prob.num_partitions)


def static_plan(prob):
    """Equal-token contiguous split of the packed context stream."""
    P, C = prob.num_partitions, prob.chunk_kv
    T = int(prob.ctx_offsets[-1])
    bounds = [(p * T) // P for p in range(P + 1)]
    pieces = []  # (b, c, lo_abs, hi_abs, p)
    for p in range(P):
        t0, t1 = bounds[p], bounds[p + 1]
        for b in range(prob.num_samples):
            k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
            for c in range((k1 - k0 + C - 1) // C):
                lo = max(t0, k0 + c * C)
                hi = min(t1, k0 + (c + 1) * C, k1)
                if hi > lo:
                    pieces.append((b, c, lo, hi, p))
    pieces.sort(key=lambda x: (x[0], x[1], x[2]))
    items = []
    prev = None
    s = 0
    for (b, c, lo, hi, p) in pieces:
        s = s + 1 if prev == (b, c) else 0
        prev = (b, c)
        for g in range(prob.num_kv_heads):
            items.append(Item(b, c, g, s, lo, hi, item_cost(prob, b, lo, hi), p))
    items.sort(key=lambda it: (it.b, it.c, it.g, it.sub))
    return items, partition_loads(items, P)


def static_loads_by_tokens(prob) -> List[int]:
    """Static partition loads straight from the token ranges (no items):
    Hq * block_q * sum over samples and anchors of |[t0, t1) ∩ [k0, k0 + a)|."""
    P = prob.num_partitions
    T = int(prob.ctx_offsets[-1])
    loads = []
    for p in range(P):
        t0, t1 = (p * T) // P, ((p + 1) * T) // P
        tot = 0
        for b in range(prob.num_samples):
            k0 = int(prob.ctx_offsets[b])
            for j in range(int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])):
                a = int(prob.anchors[j])
                tot += max(0, min(t1, k0 + a) - max(t0, k0))
        loads.append(prob.num_q_heads * prob.block_q * tot)
    return loads


def partition_loads(items: List[Item], P: int) -> List[int]:
    load = [0] * P
    for it in items:
        load[it.partition] += it.cost
    return load


def imbalance(loads: List[int]) -> float:
    """max / mean - 1 over all partitions."""
    tot = sum(loads)
    if tot == 0:
        return 0.0
    return max(loads) * len(loads) / tot - 1.0


def makespan(costs: List[int], part: List[int], P: int) -> int:
    load = [0] * P
    for c, p in zip(costs, part):
        load[p] += c
    return max(load)
