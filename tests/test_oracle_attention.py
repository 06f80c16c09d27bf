"""Pins of the attention oracle against things other than itself: a library
attention routine, autograd, finite differences, closed forms and the
exactness of the split ("Split-KV: Efficient Context Parallelism for Training
Diffusion Drafters", Abstract: exact CP; "Split-KV: Breaking the Context
Parallelism Bottleneck ...", section "Split-KV's Core Mechanism": results
strictly consistent with the unsharded case)."""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import attention as A
from split_kv_block_b200 import synth

F64 = torch.float64


def _tensors(prob, seed=0):
    return synth.make_tensors(prob, seed=seed, backward=True)


def _sdpa_reference(prob, q, k, v, requires_grad=False):
    """torch's scaled_dot_product_attention in fp64 with an explicit boolean
    mask per sample: query token t of anchor a may see context key kk iff
    kk < a. Returns O [Nq, Hq, d] (differentiable when asked)."""
    q = q.to(F64).requires_grad_(requires_grad)
    k = k.to(F64).requires_grad_(requires_grad)
    v = v.to(F64).requires_grad_(requires_grad)
    G = prob.num_q_heads // prob.num_kv_heads
    S = prob.block_q
    outs = []
    for b in range(prob.num_samples):
        k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
        j0, j1 = int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])
        if j1 == j0:
            continue
        qb = q[j0 * S:j1 * S].permute(1, 0, 2)                     # [Hq, n, d]
        kb = k[k0:k1].repeat_interleave(G, dim=1).permute(1, 0, 2)  # [Hq, L, d]
        vb = v[k0:k1].repeat_interleave(G, dim=1).permute(1, 0, 2)
        a_tok = torch.tensor(np.repeat(prob.anchors[j0:j1], S))
        mask = torch.arange(k1 - k0)[None, :] < a_tok[:, None]    # [n, L]
        if prob.key_block_mask is not None:                        # and the key's block set for the anchor
            rows = torch.from_numpy(np.repeat(prob.key_block_mask[j0:j1], S, axis=0).astype(bool))
            mask = mask & rows[:, torch.arange(k1 - k0) // 128]
        ob = F.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask)
        outs.append(ob.permute(1, 0, 2))
    return torch.cat(outs, 0), (q, k, v)


def _probs():
    rng = np.random.default_rng(7)
    yield synth.small_problem([300], [[1, 77, 300]], block_q=4, hq=4, hkv=2, d=16)
    yield synth.small_problem([130, 257], [[5, 130], [256, 1, 100]], block_q=2, hq=8, hkv=2, d=32)
    for _ in range(3):
        yield synth.random_small_problem(rng, max_len=260, max_anchors=3, d=16)


@pytest.mark.parametrize("pi", range(5))
def test_forward_matches_library_sdpa(pi):
    prob = list(_probs())[pi]
    q, k, v, _ = _tensors(prob, seed=pi)
    O, LSE = A.attention_forward(prob, q, k, v)
    ref, _ = _sdpa_reference(prob, q, k, v)
    assert torch.allclose(O, ref, atol=1e-11, rtol=0)
    assert torch.isfinite(LSE).all()


@pytest.mark.parametrize("pi", range(5))
def test_backward_matches_autograd(pi):
    prob = list(_probs())[pi]
    q, k, v, do = _tensors(prob, seed=10 + pi)
    O, LSE = A.attention_forward(prob, q, k, v)
    dq, dk, dv = A.attention_backward(prob, q, k, v, O, LSE, do)
    ref, (q64, k64, v64) = _sdpa_reference(prob, q, k, v, requires_grad=True)
    (ref * do.to(F64)).sum().backward()
    for mine, theirs in ((dq, q64.grad), (dk, k64.grad), (dv, v64.grad)):
        assert torch.allclose(mine, theirs, atol=1e-10, rtol=0)


def test_backward_central_differences():
    """d/dx of sum(O * dO), x in a few entries of q, k, v, by central
    differences of the oracle's own forward in fp64."""
    prob = synth.small_problem([40], [[7, 40]], block_q=2, hq=2, hkv=1, d=8)
    q, k, v, do = _tensors(prob, seed=3)
    q, k, v, do = q.to(F64), k.to(F64), v.to(F64), do.to(F64)
    O, LSE = A.attention_forward(prob, q, k, v)
    dq, dk, dv = A.attention_backward(prob, q, k, v, O, LSE, do)

    def loss(qq, kk, vv):
        return float((A.attention_forward(prob, qq, kk, vv)[0] * do).sum())

    eps = 1e-6
    for name, t, g, idxs in (("q", q, dq, [(0, 0, 0), (3, 1, 5)]),
                             ("k", k, dk, [(0, 0, 1), (6, 0, 7), (20, 0, 2)]),
                             ("v", v, dv, [(2, 0, 3), (39, 0, 0)])):
        for idx in idxs:
            tp, tm = t.clone(), t.clone()
            tp[idx] += eps
            tm[idx] -= eps
            args_p = {"q": (tp, k, v), "k": (q, tp, v), "v": (q, k, tp)}[name]
            args_m = {"q": (tm, k, v), "k": (q, tm, v), "v": (q, k, tm)}[name]
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - float(g[idx])) < 1e-6, (name, idx, fd, float(g[idx]))
    # keys beyond every anchor get exactly zero gradient
    assert torch.all(dk[40:] == 0) and torch.all(dv[40:] == 0)


def test_zero_queries_give_prefix_mean():
    """Q = 0: every score is 0, so LSE = ln a and O = mean of V[0:a]."""
    prob = synth.small_problem([200, 64], [[1, 50, 200], [64, 3]], block_q=3, hq=4, hkv=2, d=16)
    q, k, v, _ = _tensors(prob)
    q = torch.zeros_like(q)
    O, LSE = A.attention_forward(prob, q, k, v)
    G = 2
    for b, j, rows, k0, a in A._blocks(prob):
        assert torch.allclose(LSE[rows], torch.full_like(LSE[rows], math.log(a)), atol=1e-13)
        for h in range(4):
            mean = v[k0:k0 + a, h // G].to(F64).mean(0)
            assert torch.allclose(O[rows, h], mean.expand_as(O[rows, h]), atol=1e-13)


def test_single_key_anchor():
    """a = 1: the block sees key 0 only: O = V[0], LSE = q . k_0 / sqrt(d)."""
    d = 16
    prob = synth.small_problem([30], [[1]], block_q=4, hq=4, hkv=2, d=d)
    q, k, v, _ = _tensors(prob)
    O, LSE = A.attention_forward(prob, q, k, v)
    for h in range(4):
        g = h // 2
        assert torch.allclose(O[:, h], v[0, g].to(F64).expand(4, d), atol=0)
        s0 = (q[:, h].to(F64) * k[0, g].to(F64)).sum(-1) / math.sqrt(d)
        assert torch.allclose(LSE[:, h], s0, atol=1e-13)


def test_constant_values():
    """V constant along keys: O equals that constant; dP = dO . v = D so
    dQ = dK = 0, and dV = P^T dO."""
    prob = synth.small_problem([90], [[9, 90, 45]], block_q=2, hq=4, hkv=1, d=8)
    q, k, v, do = _tensors(prob)
    row = torch.randn(1, 1, 8, generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    v = row.expand(90, 1, 8).contiguous()
    O, LSE = A.attention_forward(prob, q, k, v)
    assert torch.allclose(O, row.to(F64).expand_as(O), atol=1e-14)
    dq, dk, dv = A.attention_backward(prob, q, k, v, O, LSE, do)
    assert dq.abs().max() < 1e-12 and dk.abs().max() < 1e-12
    assert dv.abs().max() > 1e-3


@pytest.mark.parametrize("chunk,sub", [(1, 1), (7, 1), (64, 1), (64, 4), (100, 2), (1000, 1), (4096, 8)])
def test_split_equals_unsplit(chunk, sub):
    """Exactness of the split: merge(per-chunk partials) == unsplit attention
    for any chunking, including single-key chunks and one chunk over all."""
    prob = synth.small_problem([150, 37], [[150, 3, 80], [37, 20]], block_q=2, hq=4, hkv=2, d=16,
                               chunk_kv=chunk, sub_chunks=sub)
    q, k, v, do = _tensors(prob, seed=5)
    O, LSE = A.attention_forward(prob, q, k, v)
    Oc, LSEc = A.chunked_forward(prob, q, k, v)
    assert torch.allclose(O, Oc, atol=1e-12, rtol=0)
    assert torch.allclose(LSE, LSEc, atol=1e-12, rtol=0)
    g_ref = A.attention_backward(prob, q, k, v, O, LSE, do)
    g_chk = A.chunked_backward(prob, q, k, v, Oc, LSEc, do)
    for a_, b_ in zip(g_ref, g_chk):
        assert torch.allclose(a_, b_, atol=1e-12, rtol=0)


def test_merge_of_two_halves_by_hand():
    """Two partials over disjoint key sets: LSE = ln(e^l1 + e^l2) and the
    output is the softmax-weighted average (worked by hand on numbers)."""
    o1 = torch.tensor([[[1.0, 0.0]]], dtype=F64)
    o2 = torch.tensor([[[0.0, 2.0]]], dtype=F64)
    l1 = torch.tensor([[math.log(3.0)]], dtype=F64)
    l2 = torch.tensor([[math.log(1.0)]], dtype=F64)
    dead = (torch.zeros_like(o1), torch.full_like(l1, -math.inf))
    O, L = A.lse_merge([(o1, l1), dead, (o2, l2)])
    assert abs(float(L) - math.log(4.0)) < 1e-15
    assert torch.allclose(O, torch.tensor([[[0.75, 0.5]]], dtype=F64), atol=1e-15)


def test_flops_fwd_hand_instance_and_mask_count():
    """Forward FLOPs = 4 d per unmasked (query token, key, q-head) triple.
    Hand instance: one 10-key sample, anchors 3 and 7, block_q 2, 4 q-heads,
    d 8: 2 tokens x (3 + 7) keys x 4 heads = 80 triples, 4 * 8 * 80 = 2560.
    Random ragged problems: the triples counted one by one from the explicit
    boolean mask of every sample."""
    prob = synth.small_problem([10], [[3, 7]], block_q=2, hq=4, hkv=2, d=8)
    assert A.flops_fwd(prob) == 2560
    rng = np.random.default_rng(21)
    for _ in range(20):
        prob = synth.random_small_problem(rng)
        S = prob.block_q
        triples = 0
        for b in range(prob.num_samples):
            k0, k1 = int(prob.ctx_offsets[b]), int(prob.ctx_offsets[b + 1])
            for j in range(int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])):
                for _t in range(S):
                    for kk in range(k1 - k0):
                        if kk < int(prob.anchors[j]):
                            triples += prob.num_q_heads
        assert A.flops_fwd(prob) == 4 * prob.head_dim * triples



def _masked(prob, seed, density=0.4):
    """The problem with a random block mask that leaves every anchor at least
    its first block (so no row of the library reference is empty)."""
    rng = np.random.default_rng(seed)
    lens = np.diff(prob.ctx_offsets)
    stride = int((lens.max() + 127) // 128)
    m = (rng.random((int(prob.anchor_offsets[-1]), stride)) < density).astype(np.uint8)
    m[:, 0] = 1
    return prob.replace(key_block_mask=m)


def _mask_probs():
    yield synth.small_problem([700, 390], [[650, 129, 300], [390, 200]], block_q=2, hq=4, hkv=2, d=16)
    yield synth.small_problem([1000], [[999, 513, 256, 40]], block_q=3, hq=8, hkv=2, d=16)


@pytest.mark.parametrize("pi", range(2))
def test_block_mask_forward_backward_match_library_sdpa_and_autograd(pi):
    """Block-sparse mask: forward against torch SDPA with the explicit boolean
    mask (prefix AND block bit), gradients against autograd through it."""
    prob = _masked(list(_mask_probs())[pi], seed=pi)
    q, k, v, do = _tensors(prob, seed=pi)
    O, L = A.attention_forward(prob, q, k, v)
    ref, (qq, kk, vv) = _sdpa_reference(prob, q, k, v, requires_grad=True)
    assert torch.allclose(O, ref.detach(), atol=1e-12, rtol=0)
    (ref * do.to(F64)).sum().backward()
    gq, gk, gv = A.attention_backward(prob, q, k, v, O, L, do)
    assert torch.allclose(gq, qq.grad, atol=1e-11, rtol=0)
    assert torch.allclose(gk, kk.grad, atol=1e-11, rtol=0)
    assert torch.allclose(gv, vv.grad, atol=1e-11, rtol=0)


def test_block_mask_of_ones_is_the_prefix_mask_and_block_zero_caps_the_anchor():
    """All blocks set: the prefix mask exactly. Only block 0 set: the prefix
    mask with every anchor capped at 128 (a closed form of the reading)."""
    prob = list(_mask_probs())[0]
    q, k, v, do = _tensors(prob, seed=3)
    stride = 6
    ones = prob.replace(key_block_mask=np.ones((int(prob.anchor_offsets[-1]), stride), dtype=np.uint8))
    for a_, b_ in zip(A.attention_forward(prob, q, k, v), A.attention_forward(ones, q, k, v)):
        assert torch.equal(a_, b_)
    first = np.zeros((int(prob.anchor_offsets[-1]), stride), dtype=np.uint8)
    first[:, 0] = 1
    capped = prob.replace(anchors=np.minimum(prob.anchors, 128))
    O1, L1 = A.attention_forward(prob.replace(key_block_mask=first), q, k, v)
    O2, L2 = A.attention_forward(capped, q, k, v)
    assert torch.allclose(O1, O2, atol=1e-14) and torch.allclose(L1, L2, atol=1e-14)


@pytest.mark.parametrize("chunk,sub", [(128, 1), (256, 2), (384, 3), (1024, 1)])
def test_block_mask_split_equals_unsplit(chunk, sub):
    prob = _masked(synth.small_problem([700, 390], [[650, 129, 300], [390, 200]], block_q=2, hq=4, hkv=2, d=16,
                                       chunk_kv=chunk, sub_chunks=sub), seed=11)
    q, k, v, do = _tensors(prob, seed=6)
    O, L = A.attention_forward(prob, q, k, v)
    Oc, Lc = A.chunked_forward(prob, q, k, v)
    assert torch.allclose(O, Oc, atol=1e-12, rtol=0) and torch.allclose(L, Lc, atol=1e-12, rtol=0)
    for a_, b_ in zip(A.attention_backward(prob, q, k, v, O, L, do), A.chunked_backward(prob, q, k, v, Oc, Lc, do)):
        assert torch.allclose(a_, b_, atol=1e-12, rtol=0)


def test_block_mask_empty_row():
    """An anchor whose blocks are all cleared sees no key: O = 0, LSE = -inf,
    no gradient to any key; the other blocks are as without it."""
    prob = synth.small_problem([400], [[390, 200]], block_q=2, hq=4, hkv=2, d=16)
    m = np.ones((2, 4), dtype=np.uint8)
    m[0, :] = 0
    mp = prob.replace(key_block_mask=m)
    q, k, v, do = _tensors(prob, seed=8)
    O, L = A.attention_forward(mp, q, k, v)
    assert torch.all(O[0:2] == 0) and torch.all(torch.isneginf(L[0:2]))
    alone = prob.replace(anchors=np.array([200]), anchor_offsets=np.array([0, 1], dtype=np.int32))
    O1, L1 = A.attention_forward(alone, q[2:4], k, v)
    assert torch.allclose(O[2:4], O1, atol=1e-14) and torch.allclose(L[2:4], L1, atol=1e-14)
    gq, gk, gv = A.attention_backward(mp, q, k, v, O, L, do)
    assert torch.all(gq[0:2] == 0)
    g1 = A.attention_backward(alone, q[2:4], k, v, O1, L1, do[2:4])
    assert torch.allclose(gk, g1[1], atol=1e-13) and torch.allclose(gv, g1[2], atol=1e-13)


def test_flops_fwd_with_a_block_mask_brute_force():
    prob = _masked(synth.small_problem([700, 390], [[650, 129, 300], [390, 200]], block_q=2, hq=4, hkv=2, d=16),
                   seed=5)
    m = prob.key_block_mask
    triples = 0
    for b in range(prob.num_samples):
        for j in range(int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])):
            for kk in range(int(prob.anchors[j])):
                if m[j, kk // 128]:
                    triples += prob.block_q * prob.num_q_heads
    assert A.flops_fwd(prob) == 4 * prob.head_dim * triples
