"""Thin Python binding of libskv.so (ctypes). Argument marshalling only:
planning runs in the library's C++ planner, every step of the attention in
its CUDA kernels. torch provides device memory and streams.

The library must be built (split_kv_block_b200.build); there is no fallback:
calls raise if libskv.so is missing or a call fails.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libskv.so")

SKV_PLAN_LPT = 0
SKV_PLAN_STATIC = 1
SKV_PLAN_LPT_TILES = 2          # LPT on the executed-tile cost (see include/skv.h)
SKV_PLAN_PARTIALS_BF16 = 0x100  # flag: bf16 partial outputs (see include/skv.h)
SKV_PLAN_PARTITION_QUEUES = 0x200  # flag: one work queue per partition (see include/skv.h)

# Every function include/skv.h declares.
EXPORTS = ("skv_plan_size", "skv_plan", "skv_plan_items", "skv_plan_unit_partitions", "skv_plan_stats", "skv_attn_fwd",
           "skv_attn_fwd_merged", "skv_lse_merge",
           "skv_attn_bwd", "skv_attn_bwd_deterministic", "skv_status", "skv_strerror", "skv_last_cuda_error", "skv_set_unit_timer",
           "skv_set_timing_events", "skv_attn_fwd_noalloc", "skv_noalloc_status", "skv_wait_selftest",
           "skv_plan_shard_size", "skv_plan_shard", "skv_plan_kv_layout", "skv_attn_bwd_partial", "skv_lse_combine",
           "skv_dq_combine", "skv_lpt_place_device")
SKV_NOALLOC_SCRATCH_BYTES = 32 << 20
SKV_KERNEL_FWD, SKV_KERNEL_MERGE, SKV_KERNEL_BWD = 0, 1, 2


class SkvError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn} failed: {msg} (status {code})")
        self.code = code


class _Problem(ctypes.Structure):
    _fields_ = [("num_samples", ctypes.c_int32), ("ctx_offsets", ctypes.c_void_p), ("anchor_offsets", ctypes.c_void_p),
                ("anchors", ctypes.c_void_p), ("block_q", ctypes.c_int32), ("chunk_kv", ctypes.c_int32),
                ("sub_chunks", ctypes.c_int32), ("num_partitions", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("key_block_mask", ctypes.c_void_p),
                ("mask_stride", ctypes.c_int32)]


ITEM_DTYPE = np.dtype([("b", np.int32), ("c", np.int32), ("g", np.int32), ("sub", np.int32),
                       ("key_begin", np.int64), ("key_end", np.int64), ("cost", np.int64),
                       ("partition", np.int32), ("order", np.int32), ("kv_row", np.int64)])

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m split_kv_block_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz = ctypes.c_void_p, ctypes.c_size_t
        L.skv_plan_size.argtypes = [vp, ctypes.c_int, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                    ctypes.POINTER(sz)]
        L.skv_plan.argtypes = [vp, ctypes.c_int, vp, sz, vp]
        L.skv_plan_items.argtypes = [vp, ctypes.POINTER(vp), ctypes.POINTER(sz)]
        L.skv_plan_stats.argtypes = [vp, vp, vp, vp, vp]
        L.skv_plan_unit_partitions.argtypes = [vp, vp, vp]
        L.skv_attn_fwd.argtypes = [vp, vp, vp, vp, vp, vp, sz, vp]
        L.skv_attn_fwd_merged.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.skv_lse_merge.argtypes = [vp, vp, vp, vp, vp, vp]
        L.skv_attn_bwd.argtypes = [vp] * 12 + [sz, vp]
        L.skv_attn_bwd_deterministic.argtypes = [vp] * 12 + [sz, vp]
        L.skv_status.argtypes = [vp, vp]
        L.skv_strerror.argtypes = [ctypes.c_int]
        L.skv_strerror.restype = ctypes.c_char_p
        L.skv_set_unit_timer.argtypes = [vp, vp]
        L.skv_set_timing_events.argtypes = [ctypes.c_int, vp, vp]
        L.skv_attn_fwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp]
        L.skv_noalloc_status.argtypes = [vp]
        L.skv_wait_selftest.argtypes = [vp, ctypes.c_uint64, ctypes.c_int, vp]
        L.skv_plan_shard_size.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.POINTER(sz), ctypes.POINTER(sz),
                                          ctypes.POINTER(sz), ctypes.POINTER(sz)]
        L.skv_plan_shard.argtypes = [vp, ctypes.c_int, ctypes.c_int, vp, sz, vp]
        L.skv_plan_kv_layout.argtypes = [vp, vp, vp, vp]
        L.skv_attn_bwd_partial.argtypes = [vp] * 12 + [sz, vp]
        L.skv_lse_combine.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int64, ctypes.c_int, vp, vp, vp]
        L.skv_dq_combine.argtypes = [vp, ctypes.c_int, ctypes.c_int64, vp, vp]
        L.skv_lpt_place_device.argtypes = [vp, ctypes.c_int64, ctypes.c_int32, vp, vp, vp]
        for name in EXPORTS:
            if name not in ("skv_strerror",):
                getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _check(fn: str, rc: int):
    if rc != 0:
        msg = lib().skv_strerror(rc).decode()
        if rc == 4:
            msg += f" (cuda error {lib().skv_last_cuda_error()})"
        raise SkvError(fn, rc, msg)


def _ptr(a) -> ctypes.c_void_p:
    if a is None:
        return ctypes.c_void_p(0)
    if isinstance(a, np.ndarray):
        return ctypes.c_void_p(a.ctypes.data)
    return ctypes.c_void_p(a.data_ptr())


def _stream_ptr(stream) -> ctypes.c_void_p:
    if stream is None:
        import torch
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(int(stream.cuda_stream))


class _ProblemArgs:
    """Keeps the arrays referenced by a skv_problem alive."""

    def __init__(self, prob):
        self.ctx = np.ascontiguousarray(prob.ctx_offsets, dtype=np.int64)
        self.aoff = np.ascontiguousarray(prob.anchor_offsets, dtype=np.int32)
        self.anchors = np.ascontiguousarray(prob.anchors, dtype=np.int64)
        m = getattr(prob, "key_block_mask", None)
        self.mask = None if m is None else np.ascontiguousarray(m, dtype=np.uint8)
        self.s = _Problem(len(self.ctx) - 1, self.ctx.ctypes.data, self.aoff.ctypes.data,
                          self.anchors.ctypes.data if self.anchors.size else 0, prob.block_q, prob.chunk_kv,
                          prob.sub_chunks, prob.num_partitions, prob.num_q_heads, prob.num_kv_heads, prob.head_dim,
                          self.mask.ctypes.data if self.mask is not None and self.mask.size else 0,
                          int(self.mask.shape[1]) if self.mask is not None else 0)

    def ref(self):
        return ctypes.byref(self.s)


@dataclass
class PlanSizes:
    n_items: int
    plan_bytes: int
    ws_fwd_bytes: int
    ws_bwd_bytes: int

    @property
    def ws_bytes(self) -> int:
        return max(self.ws_fwd_bytes, self.ws_bwd_bytes)


def skv_plan_size(prob, policy: int = SKV_PLAN_LPT) -> PlanSizes:
    args = _ProblemArgs(prob)
    out = [ctypes.c_size_t() for _ in range(4)]
    _check("skv_plan_size", lib().skv_plan_size(args.ref(), policy, *[ctypes.byref(o) for o in out]))
    return PlanSizes(*[o.value for o in out])


class Plan:
    """Host plan buffer written by skv_plan."""

    def __init__(self, buf: np.ndarray, loads: np.ndarray, sizes: PlanSizes, policy: int, prob):
        self.buf = buf
        self.partition_load = loads
        self.sizes = sizes
        self.policy = policy
        self.problem = prob
        self._pargs = _ProblemArgs(prob)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.buf.ctypes.data)

    @property
    def prob_ref(self):
        """The skv_problem the plan was made for (passed with the plan to every
        call that runs kernels; the library checks that they match)."""
        return self._pargs.ref()

    def items(self) -> np.ndarray:
        p, n = ctypes.c_void_p(), ctypes.c_size_t()
        _check("skv_plan_items", lib().skv_plan_items(self.ptr, ctypes.byref(p), ctypes.byref(n)))
        if n.value == 0:
            return np.zeros(0, dtype=ITEM_DTYPE)
        raw = (ctypes.c_uint8 * (n.value * ITEM_DTYPE.itemsize)).from_address(p.value)
        return np.frombuffer(raw, dtype=ITEM_DTYPE).copy()

    def unit_partitions(self):
        """(forward, backward) int32 arrays: the partition of every work unit, in
        the order the unit timer indexes its stamps."""
        st = self.stats()
        fp = np.zeros(st["n_fwd_units"], dtype=np.int32)
        bp = np.zeros(st["n_bwd_units"], dtype=np.int32)
        _check("skv_plan_unit_partitions", lib().skv_plan_unit_partitions(self.ptr, ctypes.c_void_p(fp.ctypes.data),
                                                                          ctypes.c_void_p(bp.ctypes.data)))
        return fp, bp

    def kv_layout(self):
        """(kv_rows, kv_heads, shard) of the K/V buffers the plan's kernels read."""
        r, hh, sh = ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check("skv_plan_kv_layout", lib().skv_plan_kv_layout(self.ptr, ctypes.byref(r), ctypes.byref(hh),
                                                              ctypes.byref(sh)))
        return r.value, hh.value, sh.value

    def stats(self) -> dict:
        tc, nf, nb = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        im = ctypes.c_double()
        _check("skv_plan_stats", lib().skv_plan_stats(self.ptr, ctypes.byref(tc), ctypes.byref(nf), ctypes.byref(nb),
                                                      ctypes.byref(im)))
        return {"total_cost": tc.value, "n_fwd_units": nf.value, "n_bwd_units": nb.value, "imbalance": im.value}


def skv_plan_shard_size(prob, partition: int, policy: int = SKV_PLAN_LPT) -> PlanSizes:
    args = _ProblemArgs(prob)
    out = [ctypes.c_size_t() for _ in range(4)]
    _check("skv_plan_shard_size", lib().skv_plan_shard_size(args.ref(), policy, int(partition),
                                                            *[ctypes.byref(o) for o in out]))
    return PlanSizes(*[o.value for o in out])


def skv_plan_shard(prob, partition: int, policy: int = SKV_PLAN_LPT) -> Plan:
    """Plan of one context-parallel rank: the items of partition `partition`
    of the global plan, K/V rows of its own items only (see include/skv.h)."""
    args = _ProblemArgs(prob)
    sizes = skv_plan_shard_size(prob, partition, policy)
    buf = np.empty(sizes.plan_bytes, dtype=np.uint8)
    loads = np.zeros(prob.num_partitions, dtype=np.int64)
    _check("skv_plan_shard", lib().skv_plan_shard(args.ref(), policy, int(partition), ctypes.c_void_p(buf.ctypes.data),
                                                  buf.nbytes, ctypes.c_void_p(loads.ctypes.data)))
    return Plan(buf, loads, sizes, policy, prob)


def skv_plan(prob, policy: int = SKV_PLAN_LPT, sizes: Optional[PlanSizes] = None, buf: Optional[np.ndarray] = None) -> Plan:
    args = _ProblemArgs(prob)
    if sizes is None:
        sizes = skv_plan_size(prob, policy)
    if buf is None or buf.nbytes < sizes.plan_bytes:
        buf = np.empty(sizes.plan_bytes, dtype=np.uint8)
    loads = np.zeros(prob.num_partitions, dtype=np.int64)
    _check("skv_plan", lib().skv_plan(args.ref(), policy, ctypes.c_void_p(buf.ctypes.data), buf.nbytes,
                                      ctypes.c_void_p(loads.ctypes.data)))
    return Plan(buf, loads, sizes, policy, prob)


def alloc_workspace(plan: Plan, device="cuda"):
    import torch
    return torch.empty(plan.sizes.ws_bytes, dtype=torch.uint8, device=device)


def skv_attn_fwd(plan: Plan, q, k, v, ws, stream=None):
    _check("skv_attn_fwd", lib().skv_attn_fwd(plan.ptr, plan.prob_ref, _ptr(q), _ptr(k), _ptr(v), _ptr(ws),
                                              ws.numel(), _stream_ptr(stream)))


def skv_attn_fwd_merged(plan: Plan, q, k, v, o, lse, ws, stream=None):
    """Forward and LSE merge in one launch (the merge runs in the forward's tail)."""
    _check("skv_attn_fwd_merged", lib().skv_attn_fwd_merged(plan.ptr, plan.prob_ref, _ptr(q), _ptr(k), _ptr(v),
                                                            _ptr(o), _ptr(lse), _ptr(ws), ws.numel(),
                                                            _stream_ptr(stream)))


def skv_lse_merge(plan: Plan, ws, o, lse, stream=None):
    _check("skv_lse_merge", lib().skv_lse_merge(plan.ptr, plan.prob_ref, _ptr(ws), _ptr(o), _ptr(lse),
                                                _stream_ptr(stream)))


def skv_attn_bwd(plan: Plan, q, k, v, o, lse, do, dq, dk, dv, ws, stream=None, deterministic=False):
    if deterministic:
        _check("skv_attn_bwd_deterministic", lib().skv_attn_bwd_deterministic(
            plan.ptr, plan.prob_ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk),
            _ptr(dv), _ptr(ws), ws.numel(), _stream_ptr(stream)))
        return
    _check("skv_attn_bwd", lib().skv_attn_bwd(plan.ptr, plan.prob_ref, _ptr(q), _ptr(k), _ptr(v), _ptr(o),
                                              _ptr(lse), _ptr(do), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(ws),
                                              ws.numel(), _stream_ptr(stream)))


def skv_wait_selftest(ws, limit_ns: int, arrive: bool, stream=None):
    """One bounded device-side wait of `limit_ns`: completed first (arrive) or
    never (its give-up leaves SKV_ETIMEOUT in ws's status word)."""
    _check("skv_wait_selftest", lib().skv_wait_selftest(_ptr(ws), int(limit_ns), 1 if arrive else 0,
                                                        _stream_ptr(stream)))


def skv_attn_fwd_noalloc(plan: Plan, q, k, v, o, lse, stream=None):
    """Forward + merge with the library's static scratch: for callers that
    cannot allocate device memory (see include/skv.h)."""
    _check("skv_attn_fwd_noalloc", lib().skv_attn_fwd_noalloc(plan.ptr, plan.prob_ref, _ptr(q), _ptr(k), _ptr(v),
                                                              _ptr(o), _ptr(lse), _stream_ptr(stream)))


def skv_noalloc_status(stream=None) -> int:
    """Status word of the last skv_attn_fwd_noalloc call on the current device
    (synchronizes the stream; allocates nothing)."""
    return lib().skv_noalloc_status(_stream_ptr(stream))


def skv_attn_bwd_partial(plan: Plan, q, k, v, o, lse, do, dq_f32, dk, dv, ws, stream=None):
    """Backward with dQ written in fp32 (the plan's share of dQ)."""
    _check("skv_attn_bwd_partial", lib().skv_attn_bwd_partial(plan.ptr, plan.prob_ref, _ptr(q), _ptr(k), _ptr(v),
                                                              _ptr(o), _ptr(lse), _ptr(do), _ptr(dq_f32), _ptr(dk),
                                                              _ptr(dv), _ptr(ws), ws.numel(), _stream_ptr(stream)))


def skv_lse_combine(o_parts, lse_parts, o, lse, stream=None):
    """o_parts bf16 [R, ..., d], lse_parts fp32 [R, ...] -> o, lse (rank partials combined in rank order)."""
    n_parts = int(o_parts.shape[0])
    d = int(o_parts.shape[-1])
    n_rows = int(lse_parts.numel() // n_parts)
    _check("skv_lse_combine", lib().skv_lse_combine(_ptr(o_parts), _ptr(lse_parts), n_parts, n_rows, d, _ptr(o),
                                                    _ptr(lse), _stream_ptr(stream)))


def skv_dq_combine(dq_parts, dq, stream=None):
    """dq_parts fp32 [R, ...] -> dq bf16 (sum over ranks in rank order)."""
    n_parts = int(dq_parts.shape[0])
    _check("skv_dq_combine", lib().skv_dq_combine(_ptr(dq_parts), n_parts, int(dq_parts.numel() // n_parts), _ptr(dq),
                                                  _stream_ptr(stream)))


def skv_lpt_place_device(costs, n_partitions: int, partition, loads, stream=None):
    """LPT placement on the GPU: costs int64 [n] (device), partition int32 [n]
    and loads int64 [P] (device outputs); the same bits as skv_plan's."""
    _check("skv_lpt_place_device", lib().skv_lpt_place_device(_ptr(costs), int(costs.numel()), int(n_partitions),
                                                              _ptr(partition), _ptr(loads), _stream_ptr(stream)))


def skv_status(ws, stream=None) -> int:
    return lib().skv_status(_ptr(ws), _stream_ptr(stream))


def skv_set_unit_timer(fwd_stamps=None, bwd_stamps=None):
    _check("skv_set_unit_timer", lib().skv_set_unit_timer(_ptr(fwd_stamps), _ptr(bwd_stamps)))


def skv_set_timing_events(kernel: int, start=None, end=None):
    """start/end: torch.cuda.Event (already recorded once, so the CUDA event exists) or None."""
    h0 = ctypes.c_void_p(start.cuda_event) if start is not None else ctypes.c_void_p(0)
    h1 = ctypes.c_void_p(end.cuda_event) if end is not None else ctypes.c_void_p(0)
    _check("skv_set_timing_events", lib().skv_set_timing_events(kernel, h0, h1))


# ------------------------------------------------------------- conveniences
def check_inputs(plan: Plan, q, k, v, do=None):
    """Shapes, dtype and device of the call's tensors: queries in the problem's
    layout, K/V in the plan's (the packed context, or a rank's shard rows)."""
    import torch
    p = plan.problem
    Nq = p.num_tokens_q
    rows, heads, _ = plan.kv_layout()
    for name, t, shape in (("q", q, (Nq, p.num_q_heads, p.head_dim)), ("k", k, (rows, heads, p.head_dim)),
                           ("v", v, (rows, heads, p.head_dim))) + ((("do", do, (Nq, p.num_q_heads, p.head_dim)),)
                                                                    if do is not None else ()):
        if tuple(t.shape) != shape or t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name}: expected contiguous cuda bf16 {shape}, got {tuple(t.shape)} {t.dtype} {t.device}")


def forward(plan: Plan, q, k, v, ws=None, stream=None, fused=False):
    """Split-KV forward + LSE merge: the forward and merge calls in turn (the
    default, the faster on B200), or one launch with the merge in the
    forward's tail (fused). Returns (o bf16 [Nq,Hq,d], lse fp32 [Nq,Hq])."""
    import torch
    check_inputs(plan, q, k, v)
    if ws is None:
        ws = alloc_workspace(plan, q.device)
    p = plan.problem
    o = torch.empty(p.num_tokens_q, p.num_q_heads, p.head_dim, dtype=torch.bfloat16, device=q.device)
    lse = torch.empty(p.num_tokens_q, p.num_q_heads, dtype=torch.float32, device=q.device)
    if fused:
        skv_attn_fwd_merged(plan, q, k, v, o, lse, ws, stream)
    else:
        skv_attn_fwd(plan, q, k, v, ws, stream)
        skv_lse_merge(plan, ws, o, lse, stream)
    return o, lse


def backward(plan: Plan, q, k, v, o, lse, do, ws=None, stream=None, deterministic=False):
    """Split-KV backward. Returns (dq, dk, dv) bf16. deterministic: dQ summed
    over key tiles in a fixed order (bitwise reproducible, slower)."""
    import torch
    check_inputs(plan, q, k, v, do)
    if ws is None:
        ws = alloc_workspace(plan, q.device)
    dq = torch.empty_like(q)
    dk = torch.empty_like(k)
    dv = torch.empty_like(v)
    skv_attn_bwd(plan, q, k, v, o, lse, do, dq, dk, dv, ws, stream, deterministic)
    return dq, dk, dv
