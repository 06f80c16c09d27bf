"""fp64 CPU oracle: block-sparse cross-attention of anchor blocks, split-KV form.

Test infrastructure only (see oracle/__init__.py).

The operation ([Abstract]; [Article] "Split-KV's Core Mechanism"): draft
queries are built by anchor sampling, one block of `block_q` tokens per
anchor, and cross-attend to the sample's context under a block-sparse mask.
Readings taken where the pages give no formula:
  * the block of anchor a attends to context keys [0, a) of its own sample
    (exclusive end, 1 <= a <= L); no attention among draft tokens;
  * a problem may add a block-sparse mask over the context: a byte per
    (anchor, block of 128 keys of the sample); the block of anchor j then
    attends only the keys of [0, a_j) whose block is set. A block left with
    no key gets O = 0, LSE = -inf and contributes no gradient;
  * softmax scale 1/sqrt(d); LSE is the natural log-sum-exp of the scaled
    scores;
  * grouped heads: q-head h reads kv-head h // (Hq / Hkv).
Split-KV keeps K/V chunks apart, computes a partial result per chunk for the
whole (global) query set and combines the partials with query-sized tensors;
the pages state the combination is exact, i.e. equal to unsplit attention.
The exact combination of softmax partials is the log-sum-exp merge written
out in `lse_merge`. Backward: gradients are those of the unsplit attention;
per chunk they are obtained by recomputing probabilities with the merged
(final) LSE, which gives each chunk's dK/dV exactly and dQ as a sum over
chunks.

All arithmetic is fp64 on bf16-valued inputs upcast exactly.
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np
import torch

F64 = torch.float64


def _prep(q, k, v):
    return q.to(F64), k.to(F64), v.to(F64)


def _blocks(prob):
    """Yield (b, j, token_rows slice, absolute key start of the sample, anchor a)."""
    S = prob.block_q
    for b in range(prob.num_samples):
        k0 = int(prob.ctx_offsets[b])
        for j in range(int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])):
            yield b, j, slice(j * S, (j + 1) * S), k0, int(prob.anchors[j])


MASK_BLOCK = 128


def allowed_keys(prob, j: int, a: int, lo: int = 0, hi=None, k0: int = 0):
    """Keys (absolute: sample start k0 added) the block of anchor j attends,
    within the sample-relative range [lo, hi): the prefix [0, a) and, when the
    problem carries a block-sparse mask, only the keys kk whose block kk // 128
    is set in row j of the mask (reading of the pages' "block-sparse mask over
    the context"). A slice without a mask, an index tensor with one."""
    hi = a if hi is None else min(hi, a)
    lo = max(lo, 0)
    m = getattr(prob, "key_block_mask", None)
    if m is None:
        return slice(k0 + lo, k0 + max(hi, lo))
    kk = torch.arange(lo, max(hi, lo), dtype=torch.long)
    if kk.numel():
        keep = torch.from_numpy(np.asarray(m[j])[kk.numpy() // MASK_BLOCK] != 0)
        kk = kk[keep]
    return k0 + kk


def _n_keys(keys) -> int:
    return keys.stop - keys.start if isinstance(keys, slice) else int(keys.numel())


def attention_forward(prob, q, k, v) -> Tuple[torch.Tensor, torch.Tensor]:
    """Unsplit masked attention (the definition).

    For every anchor block, q-head h (group g), token t, over keys kk in [0, a):
        s_kk = q . K[k0 + kk, g] / sqrt(d)
        LSE  = ln sum_kk exp(s_kk)          (max-subtracted)
        O    = sum_kk exp(s_kk - LSE) V[k0 + kk, g]
    Returns O [Nq, Hq, d] and LSE [Nq, Hq] in fp64.
    """
    q, k, v = _prep(q, k, v)
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    scale = 1.0 / math.sqrt(d)
    O = torch.zeros(Nq, Hq, d, dtype=F64)
    LSE = torch.zeros(Nq, Hq, dtype=F64)
    for b, j, rows, k0, a in _blocks(prob):
        keys = allowed_keys(prob, j, a, k0=k0)
        if _n_keys(keys) == 0:         # a block that may see no key: O = 0, LSE = -inf
            LSE[rows] = -math.inf
            continue
        for h in range(Hq):
            g = h // G
            Kb, Vb = k[keys, g], v[keys, g]
            s = (q[rows, h] @ Kb.T) * scale                  # [S, n_keys]
            m = s.max(dim=1, keepdim=True).values
            e = torch.exp(s - m)
            l = e.sum(dim=1, keepdim=True)
            LSE[rows, h] = (m + torch.log(l)).squeeze(1)
            O[rows, h] = (e / l) @ Vb
    return O, LSE


def attention_backward(prob, q, k, v, o, lse, do):
    """Gradients of the unsplit masked attention, fp64.

        D    = sum_d dO * O                       per (token, head)
        P_kk = exp(s_kk - LSE)
        dS   = P * (dO . V[kk] - D)
        dQ   = sum_kk dS_kk K[kk] / sqrt(d)
        dK[kk, g] += dS_kk q / sqrt(d),  dV[kk, g] += P_kk dO   (summed over the
                                                               q-heads of group g)
    Keys no block attends to get zero gradients.
    """
    q, k, v = _prep(q, k, v)
    o, lse, do = o.to(F64), lse.to(F64), do.to(F64)
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    scale = 1.0 / math.sqrt(d)
    D = (do * o).sum(dim=-1)
    dq = torch.zeros_like(q)
    dk = torch.zeros_like(k)
    dv = torch.zeros_like(v)
    for b, j, rows, k0, a in _blocks(prob):
        keys = allowed_keys(prob, j, a, k0=k0)
        if _n_keys(keys) == 0:
            continue
        for h in range(Hq):
            g = h // G
            Kb, Vb = k[keys, g], v[keys, g]
            s = (q[rows, h] @ Kb.T) * scale
            P = torch.exp(s - lse[rows, h][:, None])
            dP = do[rows, h] @ Vb.T
            dS = P * (dP - D[rows, h][:, None])
            dq[rows, h] += (dS @ Kb) * scale
            dk[keys, g] += (dS.T @ q[rows, h]) * scale
            dv[keys, g] += P.T @ do[rows, h]
    return dq, dk, dv


# ------------------------------------------------------------- split-KV form
def chunk_partial(prob, q, k, v, b: int, key_begin: int, key_end: int):
    """Partial attention of every query block of sample b over the absolute
    key range [key_begin, key_end) (one KV chunk or sub-chunk), fp64.

    Returns (O_c [Nq, Hq, d], LSE_c [Nq, Hq]); rows with no unmasked key in
    the range (and rows of other samples) get LSE_c = -inf and O_c = 0.
    """
    q, k, v = _prep(q, k, v)
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    scale = 1.0 / math.sqrt(d)
    O = torch.zeros(Nq, Hq, d, dtype=F64)
    LSE = torch.full((Nq, Hq), -math.inf, dtype=F64)
    for bb, j, rows, k0, a in _blocks(prob):
        if bb != b:
            continue
        keys = allowed_keys(prob, j, a, key_begin - k0, key_end - k0, k0=k0)
        if _n_keys(keys) == 0:
            continue
        for h in range(Hq):
            g = h // G
            s = (q[rows, h] @ k[keys, g].T) * scale
            m = s.max(dim=1, keepdim=True).values
            e = torch.exp(s - m)
            l = e.sum(dim=1, keepdim=True)
            LSE[rows, h] = (m + torch.log(l)).squeeze(1)
            O[rows, h] = (e / l) @ v[keys, g]
    return O, LSE


def lse_merge(partials: Sequence[Tuple[torch.Tensor, torch.Tensor]]):
    """Exact combination of softmax partials, per (query, head):
        m   = max_c LSE_c
        LSE = m + ln sum_c exp(LSE_c - m)
        O   = sum_c exp(LSE_c - LSE) O_c
    Partials with LSE_c = -inf contribute nothing. Summation runs over the
    given order.
    """
    lses = torch.stack([p[1] for p in partials])            # [C, Nq, Hq]
    m = lses.max(dim=0).values
    m_safe = torch.where(torch.isfinite(m), m, torch.zeros_like(m))
    w = torch.exp(lses - m_safe[None])                       # exp(-inf) = 0
    lse = m_safe + torch.log(w.sum(dim=0))
    O = torch.zeros_like(partials[0][0])
    for (o_c, l_c) in partials:
        O += torch.exp(l_c - lse)[..., None] * o_c
    return O, lse


def split_ranges(prob, chunk_kv: int, sub_chunks: int = 1) -> List[Tuple[int, int, int]]:
    """(b, key_begin, key_end) absolute ranges of every chunk / sub-chunk:
    chunk c of sample b is [c*C, min((c+1)*C, L_b)); sub-chunk s of it is
    [c*C + s*C/sub, min(c*C + (s+1)*C/sub, chunk end)); empty pieces dropped."""
    out = []
    cs = chunk_kv // sub_chunks
    for b in range(prob.num_samples):
        k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
        L = k1 - k0
        for c in range((L + chunk_kv - 1) // chunk_kv):
            c_end = min((c + 1) * chunk_kv, L)
            for s in range(sub_chunks):
                lo, hi = c * chunk_kv + s * cs, min(c * chunk_kv + (s + 1) * cs, c_end)
                if hi > lo:
                    out.append((b, k0 + lo, k0 + hi))
    return out


def chunked_forward(prob, q, k, v, ranges=None):
    """Split-KV forward: a partial per key range, then the LSE merge.
    Ranges default to the problem's chunks/sub-chunks, merged in ascending
    key order."""
    if ranges is None:
        ranges = split_ranges(prob, prob.chunk_kv, prob.sub_chunks)
    parts = [chunk_partial(prob, q, k, v, b, lo, hi) for (b, lo, hi) in ranges]
    return lse_merge(parts)


def chunked_backward(prob, q, k, v, o, lse, do, ranges=None):
    """Split-KV backward: per key range, probabilities recomputed with the
    merged LSE and D = dO . O; dK/dV of the range are written by that range
    alone, dQ partials are summed over ranges in ascending key order."""
    if ranges is None:
        ranges = split_ranges(prob, prob.chunk_kv, prob.sub_chunks)
    q, k, v = _prep(q, k, v)
    o, lse, do = o.to(F64), lse.to(F64), do.to(F64)
    Nq, Hq, d = q.shape
    G = Hq // k.shape[1]
    scale = 1.0 / math.sqrt(d)
    D = (do * o).sum(dim=-1)
    dk = torch.zeros_like(k)
    dv = torch.zeros_like(v)
    dq_parts = []
    for (b, lo_r, hi_r) in ranges:
        dq_c = torch.zeros_like(q)
        for bb, j, rows, k0, a in _blocks(prob):
            if bb != b:
                continue
            keys = allowed_keys(prob, j, a, lo_r - k0, hi_r - k0, k0=k0)
            if _n_keys(keys) == 0:
                continue
            for h in range(Hq):
                g = h // G
                Kc, Vc = k[keys, g], v[keys, g]
                P = torch.exp((q[rows, h] @ Kc.T) * scale - lse[rows, h][:, None])
                dS = P * (do[rows, h] @ Vc.T - D[rows, h][:, None])
                dq_c[rows, h] += (dS @ Kc) * scale
                dk[keys, g] += (dS.T @ q[rows, h]) * scale
                dv[keys, g] += P.T @ do[rows, h]
        dq_parts.append(dq_c)
    dq = torch.zeros_like(q)
    for p in dq_parts:
        dq += p
    return dq, dk, dv


# ------------------------------------------------------------ small helpers
def flops_fwd(prob) -> int:
    """Unmasked forward FLOPs: 2 contractions of d per (query, key) pair and
    q-head: 4 * d * block_q * Hq * (sum over anchors of their attended keys;
    sum(a) without a block mask)."""
    if getattr(prob, "key_block_mask", None) is None:
        n = int(np.sum(prob.anchors))
    else:
        n = sum(_n_keys(allowed_keys(prob, j, a)) for _b, j, _r, _k0, a in _blocks(prob))
    return 4 * prob.head_dim * prob.block_q * prob.num_q_heads * n
