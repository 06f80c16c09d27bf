"""Split-KV context parallelism across GPUs: one process per GPU, the plan's P
partitions are the P ranks ("Split-KV: Breaking the Context Parallelism
Bottleneck in Diffusion Drafter Training", section "Split-KV's Core Mechanism:
Decoupling Communication from Context Length"; "Split-KV: Efficient Context
Parallelism for Training Diffusion Drafters", Abstract).

Every rank keeps the key/value rows of its own LPT items and sees the whole
query set (queries are short, so they are simply replicated: the global query
view). Per attention call only query-sized tensors cross ranks:

  forward   each rank: skv_attn_fwd + skv_lse_merge on its shard plan -> (O_r, LSE_r)
            all-gather of (O_r, LSE_r)                     [NCCL over NVLink]
            skv_lse_combine over the gathered partials      -> O, LSE on every rank
  backward  each rank: skv_attn_bwd_partial on its shard    -> fp32 dQ share, dK/dV of its rows
            all-gather of the dQ shares                     [NCCL]
            skv_dq_combine (sum in rank order, bf16)        -> dQ on every rank
            dK, dV never leave the rank.

This module moves data between ranks with torch.distributed and calls the
library for everything else; it does no arithmetic of the method. The
exchange steps are separate functions (`gather_partials`, `gather_dq`) so that
their bookkeeping can be checked with the gloo backend on CPU.
"""
from __future__ import annotations

from typing import Optional

import numpy as np
import torch
import torch.distributed as dist

from . import skv


def gather_partials(o_r: torch.Tensor, lse_r: torch.Tensor, group=None):
    """All-gather of every rank's partial output and LSE: returns
    (o_all [R, *o_r.shape], lse_all [R, *lse_r.shape]), rank r's at index r."""
    world = dist.get_world_size(group)
    o_list = [torch.empty_like(o_r) for _ in range(world)]
    l_list = [torch.empty_like(lse_r) for _ in range(world)]
    dist.all_gather(o_list, o_r.contiguous(), group=group)
    dist.all_gather(l_list, lse_r.contiguous(), group=group)
    return torch.stack(o_list), torch.stack(l_list)


def gather_dq(dq_r: torch.Tensor, group=None):
    """All-gather of every rank's fp32 dQ share: [R, *dq_r.shape], rank order."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(dq_r) for _ in range(world)]
    dist.all_gather(parts, dq_r.contiguous(), group=group)
    return torch.stack(parts)


def shard_rows(plan: skv.Plan):
    """(item rows) of a shard plan: for every item of this rank, its kv head g,
    global key range [key_begin, key_end) and first row in the shard buffers.
    Lets a data loader place the rank's K/V rows (one kv head per row)."""
    it = plan.items()
    mine = it[it["kv_row"] >= 0]
    return [(int(r["g"]), int(r["key_begin"]), int(r["key_end"]), int(r["kv_row"])) for r in mine]


def shard_kv(plan: skv.Plan, k_full: torch.Tensor) -> torch.Tensor:
    """Rows of this rank's items from a full [Ltot, Hkv, d] tensor, in the
    shard layout [kv_rows, 1, d] (data placement only, for loaders and tests)."""
    rows, _, _ = plan.kv_layout()
    out = torch.empty(rows, 1, k_full.shape[-1], dtype=k_full.dtype, device=k_full.device)
    for g, kb, ke, row in shard_rows(plan):
        out[row:row + (ke - kb), 0].copy_(k_full[kb:ke, g])
    return out


class SplitKVContextParallel:
    """One rank of a Split-KV context-parallel attention layer.

    prob.num_partitions must equal the world size: partition p of the LPT plan
    is rank p. Every rank builds the same global plan (the planner is
    deterministic) and keeps its own shard of it."""

    def __init__(self, prob, policy: int = skv.SKV_PLAN_LPT, group=None):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if prob.num_partitions != self.world:
            raise ValueError(f"num_partitions {prob.num_partitions} != world size {self.world}: "
                             "the plan's partitions are the ranks")
        self.prob = prob
        self.plan = skv.skv_plan_shard(prob, self.rank, policy)
        self.ws: Optional[torch.Tensor] = None

    def _workspace(self, device):
        if self.ws is None or self.ws.device != device:
            self.ws = skv.alloc_workspace(self.plan, device)
        return self.ws

    def forward(self, q, k_shard, v_shard, stream=None):
        """q: the full query set [Nq, Hq, d]; k_shard, v_shard: this rank's rows
        [kv_rows, 1, d]. Returns the exact O [Nq, Hq, d] and LSE [Nq, Hq],
        identical on every rank."""
        ws = self._workspace(q.device)
        o_r, lse_r = skv.forward(self.plan, q, k_shard, v_shard, ws, stream=stream, fused=False)
        o_all, lse_all = gather_partials(o_r, lse_r, self.group)
        o = torch.empty_like(o_r)
        lse = torch.empty_like(lse_r)
        skv.skv_lse_combine(o_all, lse_all, o, lse, stream)
        return o, lse

    def backward(self, q, k_shard, v_shard, o, lse, do, stream=None):
        """Returns dQ (bf16, the full query set, identical on every rank) and
        dK, dV of this rank's rows [kv_rows, 1, d]."""
        ws = self._workspace(q.device)
        dq_r = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        dk = torch.empty_like(k_shard)
        dv = torch.empty_like(v_shard)
        skv.skv_attn_bwd_partial(self.plan, q, k_shard, v_shard, o, lse, do, dq_r, dk, dv, ws, stream)
        parts = gather_dq(dq_r, self.group)
        dq = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
        skv.skv_dq_combine(parts, dq, stream)
        return dq, dk, dv
