"""Seeded synthetic inputs for split-KV attention: anchors, packed Q/K/V/dO.

This module holds no arithmetic of the method (no masking, no attention, no
cost model): it only draws random numbers and lays them out. Both the CUDA
path's tests/bench and the CPU oracle's tests take their inputs from here.

The workloads follow the regime of "Split-KV: Efficient Context Parallelism
for Training Diffusion Drafters" (Abstract): anchor sampling builds short
draft-query blocks (block_q tokens per anchor) that cross-attend to a much
longer context. The pages give no shapes; the five workloads below are the
published problem set of this project (context lengths, anchor
distributions, head counts, chunk sizes and partition counts as stated in
each entry).

Recipe (all seeded):
  * anchors come from numpy.random.default_rng(seed):
      - "uniform"   : distinct integers drawn without replacement from
                      [L // 8, L), sorted ascending;
      - "beta51"    : clip(floor(Beta(5, 1) * L), 1, L), sorted ascending
                      (duplicates possible);
  * per-sample context lengths of the batched workload are
    floor(exp(U(ln 8192, ln 262144))) from the same generator, drawn before
    the anchors;
  * Q, K, V, dO are torch.randn(..., generator=Generator().manual_seed(
    seed * 10 + k)) in fp32 for k = 0, 1, 2, 3 respectively, rounded to
    bfloat16 (round-to-nearest-even). N(0, 1) entries.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    ctx_lens: Optional[tuple]      # fixed per-sample context lengths, or None (drawn)
    num_samples: int
    anchors_per_sample: int
    anchor_dist: str               # "uniform" | "beta51"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_q: int
    chunk_kv: int
    num_partitions: int
    sub_chunks: int = 1
    backward: bool = True
    anchor_low: Optional[int] = None  # lower bound of the uniform range (default L // 8)
    mask: Optional[str] = None        # "sink_window_random": block_mask_sink_window_random(seed) on top


WORKLOADS = {
    # 1 sample, 4K context, 4 anchors in [512, 4096) x 16 tokens, 8/2 heads, d=64.
    "tiny_4k": Workload("tiny_4k", (4096,), 1, 4, "uniform", 8, 2, 64, 16, 512, 4,
                        backward=False, anchor_low=512),
    # 1 sample, 32K context, 32 anchors x 16 tokens, 32/8 heads (GQA), d=128.
    "ctx32k_fwd": Workload("ctx32k_fwd", (32768,), 1, 32, "uniform", 32, 8, 128, 16, 2048, 16,
                           backward=False),
    # same shapes with the backward pass.
    "ctx32k": Workload("ctx32k", (32768,), 1, 32, "uniform", 32, 8, 128, 16, 2048, 16),
    # 1 sample, 128K context, 64 Beta(5,1)-skewed anchors x 16 tokens.
    "ctx128k": Workload("ctx128k", (131072,), 1, 64, "beta51", 32, 8, 128, 16, 4096, 64),
    # 8 samples, context lengths log-uniform in [8192, 262144], 128 anchors each.
    "batch8_logu": Workload("batch8_logu", None, 8, 128, "uniform", 32, 8, 128, 16, 4096, 128),
    # the 32K shapes under a block-sparse mask: per anchor the first 2 key blocks of 128, the 4 blocks up
    # to its own, and each other block with probability 1/4.
    "ctx32k_sparse": Workload("ctx32k_sparse", (32768,), 1, 32, "uniform", 32, 8, 128, 16, 2048, 16,
                              mask="sink_window_random"),
}


@dataclasses.dataclass
class Problem:
    """Host description of one split-KV problem (mirrors skv_problem)."""
    ctx_offsets: np.ndarray       # int64 [B+1]
    anchor_offsets: np.ndarray    # int32 [B+1]
    anchors: np.ndarray           # int64 [A_total], 1 <= a <= L_b
    block_q: int
    chunk_kv: int
    sub_chunks: int
    num_partitions: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    # optional block-sparse mask: uint8 [A_total, mask_stride]; entry (j, kb) != 0 lets the block of anchor
    # j see keys [128 kb, 128 kb + 128) of its sample (on top of the prefix [0, a_j)); None = prefix only
    key_block_mask: Optional[np.ndarray] = None

    @property
    def num_samples(self) -> int:
        return len(self.ctx_offsets) - 1

    @property
    def num_tokens_q(self) -> int:
        return int(self.anchor_offsets[-1]) * self.block_q

    @property
    def num_tokens_kv(self) -> int:
        return int(self.ctx_offsets[-1])

    def replace(self, **kw) -> "Problem":
        return dataclasses.replace(self, **kw)


def draw_anchors(rng: np.random.Generator, L: int, n: int, dist: str, low: Optional[int] = None) -> np.ndarray:
    if dist == "uniform":
        lo = L // 8 if low is None else low
        if n > L - lo:
            raise ValueError("more anchors than distinct positions")
        a = rng.choice(np.arange(lo, L, dtype=np.int64), size=n, replace=False)
    elif dist == "beta51":
        a = np.clip(np.floor(rng.beta(5.0, 1.0, size=n) * L).astype(np.int64), 1, L)
    else:
        raise ValueError(dist)
    return np.sort(a).astype(np.int64)


def make_problem(w: Workload, seed: int = 0, *, sub_chunks: Optional[int] = None,
                 num_partitions: Optional[int] = None) -> Problem:
    rng = np.random.default_rng(seed)
    if w.ctx_lens is not None:
        lens = list(w.ctx_lens)
    else:
        lens = [int(math.floor(math.exp(rng.uniform(math.log(8192), math.log(262144)))))
                for _ in range(w.num_samples)]
    anchors = [draw_anchors(rng, L, w.anchors_per_sample, w.anchor_dist, w.anchor_low) for L in lens]
    ctx_off = np.zeros(len(lens) + 1, dtype=np.int64)
    ctx_off[1:] = np.cumsum(lens)
    anc_off = np.zeros(len(lens) + 1, dtype=np.int32)
    anc_off[1:] = np.cumsum([len(a) for a in anchors])
    p = Problem(ctx_off, anc_off, np.concatenate(anchors).astype(np.int64), w.block_q, w.chunk_kv,
                w.sub_chunks if sub_chunks is None else sub_chunks,
                w.num_partitions if num_partitions is None else num_partitions,
                w.num_q_heads, w.num_kv_heads, w.head_dim)
    if w.mask == "sink_window_random":
        p = p.replace(key_block_mask=block_mask_sink_window_random(p, seed))
    return p


def redraw_anchors(p: Problem, w: Workload, seed: int) -> Problem:
    """Same contexts, fresh anchors (one training step's anchor sampling)."""
    rng = np.random.default_rng(seed)
    lens = np.diff(p.ctx_offsets)
    anchors = [draw_anchors(rng, int(L), w.anchors_per_sample, w.anchor_dist, w.anchor_low) for L in lens]
    p = p.replace(anchors=np.concatenate(anchors).astype(np.int64))
    if w.mask == "sink_window_random":
        p = p.replace(key_block_mask=block_mask_sink_window_random(p, seed))
    return p


def randn_bf16(shape, seed: int, k: int) -> torch.Tensor:
    g = torch.Generator(device="cpu").manual_seed(seed * 10 + k)
    return torch.randn(*shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_tensors(p: Problem, seed: int = 0, backward: bool = True):
    """Packed bf16 CPU tensors: q [Nq,Hq,d], k/v [L,Hkv,d], do [Nq,Hq,d] (or None)."""
    Nq, L = p.num_tokens_q, p.num_tokens_kv
    q = randn_bf16((Nq, p.num_q_heads, p.head_dim), seed, 0)
    k = randn_bf16((L, p.num_kv_heads, p.head_dim), seed, 1)
    v = randn_bf16((L, p.num_kv_heads, p.head_dim), seed, 2)
    do = randn_bf16((Nq, p.num_q_heads, p.head_dim), seed, 3) if backward else None
    return q, k, v, do


def small_problem(lens: List[int], anchors: List[List[int]], *, block_q=16, chunk_kv=128, sub_chunks=1,
                  num_partitions=4, hq=4, hkv=1, d=64) -> Problem:
    """Hand-specified problem (tests)."""
    ctx_off = np.zeros(len(lens) + 1, dtype=np.int64)
    ctx_off[1:] = np.cumsum(lens)
    anc_off = np.zeros(len(lens) + 1, dtype=np.int32)
    anc_off[1:] = np.cumsum([len(a) for a in anchors])
    flat = np.array([x for a in anchors for x in a], dtype=np.int64)
    return Problem(ctx_off, anc_off, flat, block_q, chunk_kv, sub_chunks, num_partitions, hq, hkv, d)


def random_small_problem(rng: np.random.Generator, *, max_samples=3, max_len=700, max_anchors=5,
                         heads=((4, 1), (8, 2), (4, 4), (8, 1)), d=64) -> Problem:
    """Random ragged problem for parity sweeps: any anchor order, duplicates allowed."""
    B = int(rng.integers(1, max_samples + 1))
    lens = [int(rng.integers(1, max_len + 1)) for _ in range(B)]
    anchors = []
    for L in lens:
        n = int(rng.integers(1, max_anchors + 1))
        anchors.append([int(x) for x in rng.integers(1, L + 1, size=n)])
    hq, hkv = heads[int(rng.integers(0, len(heads)))]
    chunk = int(rng.choice([64, 128, 192, 256, 384]))
    sub = int(rng.choice([1, 2, 4])) if chunk % 4 == 0 else 1
    return small_problem(lens, anchors, block_q=int(rng.choice([1, 4, 16])), chunk_kv=chunk, sub_chunks=sub,
                         num_partitions=int(rng.integers(1, 9)), hq=hq, hkv=hkv, d=d)


MASK_BLOCK = 128  # keys per block of the block-sparse mask


def block_mask_sink_window_random(p: Problem, seed: int, sink: int = 2, window: int = 4, density: float = 0.25,
                                  ) -> np.ndarray:
    """A block-sparse mask over the context: for every anchor, the first `sink`
    key blocks of its sample, the `window` blocks ending at the one that holds
    its anchor, and each other block with probability `density` (numpy
    default_rng(seed)). Returns uint8 [A_total, stride], stride = the largest
    sample's block count."""
    rng = np.random.default_rng(seed)
    lens = np.diff(p.ctx_offsets)
    stride = int((lens.max() + MASK_BLOCK - 1) // MASK_BLOCK)
    A = int(p.anchor_offsets[-1])
    m = (rng.random((A, stride)) < density).astype(np.uint8)
    for b in range(p.num_samples):
        for j in range(int(p.anchor_offsets[b]), int(p.anchor_offsets[b + 1])):
            last = (int(p.anchors[j]) - 1) // MASK_BLOCK
            m[j, :sink] = 1
            m[j, max(0, last - window + 1):last + 1] = 1
    return m
