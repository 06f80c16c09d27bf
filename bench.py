"""Benchmark of the split-KV hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
host planning (realized cost + LPT, skv_plan), split-KV forward, LSE merge,
backward (preprocess, main kernel, dQ cast). Default workload: the 32K
context fwd+bwd problem (1 sample, 32768-token context, 32 anchors x 16 draft
tokens, 32 q / 8 kv heads, d = 128, KV chunk 2048, 16 partitions).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...     # the CPU fp64 oracle, timed on host cores

Prints one JSON line (rank 0). Multi-GPU (torchrun): every rank runs its own
independent problem (seed + rank); no data-path collective; value is the
whole-job throughput over the max-over-ranks device time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from split_kv_block_b200 import synth  # noqa: E402

WORKLOAD_TEXT = {
    "tiny_4k": "1 sample, 4096-token context, 4 anchors x 16 draft tokens, 8/2 heads, d=64, KV chunk 512, 4 partitions",
    "ctx32k_fwd": "1 sample, 32768-token context, 32 anchors x 16 draft tokens, 32/8 heads, d=128, KV chunk 2048, "
                  "16 partitions, forward + LSE merge",
    "ctx32k": "1 sample, 32768-token context, 32 anchors x 16 draft tokens, 32/8 heads, d=128, KV chunk 2048, "
              "16 partitions, fwd+bwd",
    "ctx128k": "1 sample, 131072-token context, 64 Beta(5,1) anchors x 16 draft tokens, 32/8 heads, d=128, "
               "KV chunk 4096, 64 partitions, fwd+bwd",
    "batch8_logu": "8 samples, contexts log-uniform in [8192, 262144], 128 anchors x 16 draft tokens each, 32/8 heads, "
                   "d=128, KV chunk 4096, 128 partitions, fwd+bwd, anchors redrawn and replanned every step",
    "ctx32k_sparse": "the ctx32k shapes under a block-sparse mask (per anchor: the first 2 blocks of 128 keys, the 4 "
                     "blocks up to its own, each other block with probability 1/4), fwd+bwd",
}
METRIC = "split-KV attn fwd+bwd effective TFLOP/s"
L2_BYTES = 126 * 1000 * 1000


def check_world(gpus, world):
    """--gpus N must match the number of ranks: N > 1 runs one process per GPU
    under torchrun (WORLD_SIZE = N), N = 1 a single process."""
    if gpus < 1:
        raise SystemExit(f"--gpus {gpus}: need at least one GPU")
    if gpus != world:
        raise SystemExit(f"--gpus {gpus} but WORLD_SIZE={world}: launch N > 1 with "
                         "torch.distributed.run --nproc-per-node N (one rank per GPU)")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def rank_problem(args, rank):
    """Replicas: every rank runs its own independent problem of the workload,
    seeded seed + rank (no data is shared between ranks)."""
    seed = args.seed + rank
    return seed, synth.make_problem(synth.WORKLOADS[args.workload], seed=seed, sub_chunks=args.sub_chunks)


def max_over_ranks(seconds, world, device):
    """The job's time: the maximum of the ranks' device times (all ranks call it)."""
    if world <= 1:
        return seconds
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device):
    """Sum of a per-rank quantity over all ranks (all ranks call it)."""
    if world <= 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def job_value(flops_all_ranks, seconds):
    """Whole-job throughput in TFLOP/s: the work all ranks processed (their
    problems differ, seed + rank) over the max-over-ranks time."""
    return flops_all_ranks / seconds / 1e12


def attended_keys(prob):
    """Keys every anchor's block attends, summed over anchors: sum(a) under the
    prefix mask; with a block-sparse mask, per anchor the keys of its set
    128-key blocks that lie before a."""
    m = getattr(prob, "key_block_mask", None)
    if m is None:
        return float(np.sum(prob.anchors))
    a = np.asarray(prob.anchors, dtype=np.int64)[:, None]
    starts = 128 * np.arange(m.shape[1], dtype=np.int64)[None, :]
    per_block = np.clip(a - starts, 0, 128)
    return float(((m != 0) * per_block).sum())


def flops_of(prob, backward=True):
    """Unmasked work: 4 d block_q Hq per attended key of every anchor forward
    (4 d block_q Hq sum(a) under the prefix mask), 2.5x that backward."""
    f_fwd = 4.0 * prob.head_dim * prob.block_q * prob.num_q_heads * attended_keys(prob)
    return f_fwd, (2.5 * f_fwd if backward else 0.0)


def bwd_bytes(prob):
    """Algorithmic HBM bytes of the backward attention kernel: Q, dO, LSE, D
    read once, K/V of the attended prefix read once, dK/dV of that prefix
    written once, dQ accumulated once (fp32 read + write)."""
    Nq, Hq, Hkv, d = prob.num_tokens_q, prob.num_q_heads, prob.num_kv_heads, prob.head_dim
    keys = 0
    for b in range(prob.num_samples):
        j0, j1 = int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])
        if j1 > j0:
            keys += int(prob.anchors[j0:j1].max())
    return 2 * Nq * Hq * d * 2 + 2 * Nq * Hq * 4 + 4 * keys * Hkv * d * 2 + 2 * Nq * Hq * d * 4


KERNEL_SOURCES = {"fwd_kernel": ["fwd.cu", "fwd2.cu", "sm100.cuh", "kernels.h", "plan_layout.h", "merge_row.cuh",
                                  "tail_merge.cuh"],
                  "bwd_kernel": ["bwd.cu", "bwd2.cu", "sm100.cuh", "kernels.h", "plan_layout.h"],
                  "merge_kernel": ["merge.cu", "sm100.cuh", "kernels.h", "plan_layout.h", "merge_row.cuh"]}


def kernel_digest(kernel):
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "split_kv_block_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel, workload, setup=None):
    """DRAM bytes (read + write) per launch from the committed ncu summary,
    or None when the kernel's sources changed since that capture, or when the
    run's setup (policy, partials, queues, merge, sub-chunks) differs from the
    captured one."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel, {}).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_digest") != kernel_digest(kernel):
        return None
    if setup is not None and rec.get("setup") is not None and rec["setup"] != setup:
        return None
    return rec.get("dram_bytes_per_launch")


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.rows = []
        if self.proc is None:
            return False
        time.sleep(0.1)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) == 7:
                self.rows.append(parts)
        return False

    def summary(self):
        if not getattr(self, "rows", None):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[0]) for r in self.rows if num(r[0]) is not None]
        mx = [num(r[1]) for r in self.rows if num(r[1]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in self.rows for i in range(4) if r[3 + i].lower() == "active"})
        loaded = [s for s in sm if s >= 0.5 * max(sm)] if sm else []
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(self.rows)}


# ------------------------------------------------------------- GPU arm
# Beside the headline on one GPU: (workload, LPT sub-chunks or None for the workload's own). The 128K
# workload is also timed with its chunks split in four, the granularity at which its plan is within 1 %;
# tiny_4k runs the head_dim-64 kernels.
EXTRA_WORKLOADS = (("ctx128k", None), ("ctx128k", 4), ("batch8_logu", None), ("ctx32k_sparse", None), ("tiny_4k", None))


def merge_bytes(prob, n_fwd_units):
    """Algorithmic bytes of the LSE merge kernel: every partial read once (fp32
    output row and LSE per query-tile row), merged O (bf16) and LSE (fp32)
    written once."""
    rows = prob.num_tokens_q * prob.num_q_heads
    return n_fwd_units * 128 * (prob.head_dim + 1) * 4 + rows * prob.head_dim * 2 + rows * 4


def run_workload(args, name, steps, warmup, rank, world, local_rank, e2e, sub_chunks=None):
    """Time `steps` whole steps of workload `name` (after `warmup` untimed ones)
    on this rank's GPU and return its record. sub_chunks: the LPT item split
    (None: --sub-chunks for the headline workload, the workload's own
    otherwise)."""
    from split_kv_block_b200 import skv

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = synth.WORKLOADS[name]
    seed = args.seed + rank
    if sub_chunks is None and name == args.workload:
        sub_chunks = args.sub_chunks
    prob = synth.make_problem(w, seed=seed, sub_chunks=sub_chunks)
    backward = w.backward
    q, k, v, do = synth.make_tensors(prob, seed=seed, backward=backward)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    do = do.to(dev) if backward else None
    policy = {"static": skv.SKV_PLAN_STATIC, "lpt": skv.SKV_PLAN_LPT, "lpt_tiles": skv.SKV_PLAN_LPT_TILES}[args.policy]
    if args.partials == "bf16":
        policy |= skv.SKV_PLAN_PARTIALS_BF16
    if args.queues == "partition":
        policy |= skv.SKV_PLAN_PARTITION_QUEUES
    redraw = name == "batch8_logu"
    fused = args.fused_merge  # the merge in the forward kernel's tail, or its own launch (default: faster here)
    # what a DRAM-traffic capture of this workload must have run with to stand for this run
    setup = {"policy": args.policy, "partials": args.partials, "queues": args.queues,
             "merge": "fused" if fused else "separate", "sub_chunks": prob.sub_chunks}

    # anchors of every step (the batched workload redraws them each step)
    step_probs = [synth.redraw_anchors(prob, w, seed * 1000 + i) if redraw else prob for i in range(warmup + steps)]
    sizes = [skv.skv_plan_size(p, policy) for p in step_probs]
    ws_bytes = max(s.ws_bytes for s in sizes)
    plan_bytes = max(s.plan_bytes for s in sizes)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    plan_buf = np.empty(plan_bytes, dtype=np.uint8)
    Nq, Hq, d = prob.num_tokens_q, prob.num_q_heads, prob.head_dim
    o = torch.empty(Nq, Hq, d, dtype=torch.bfloat16, device=dev)
    lse = torch.empty(Nq, Hq, dtype=torch.float32, device=dev)
    dq = dk = dv = None
    if backward:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)  # > 126 MB L2
    stream = torch.cuda.current_stream()
    # Every forward and backward call clears the workspace's status word before it runs, so the word is
    # copied (4 bytes, device to device, on the launch stream) after the merge and after the backward of
    # every step, warm-up and timed; a wait that gave up in any call is then seen after the loop.
    ws_status = ws[:4].view(torch.int32)
    status_log = torch.zeros(2 * (warmup + steps), dtype=torch.int32, device=dev)

    planner_s = []

    def step(i):
        p = step_probs[i]
        t0 = time.perf_counter()
        plan = skv.skv_plan(p, policy, sizes=sizes[i], buf=plan_buf)
        planner_s.append(time.perf_counter() - t0)
        if fused:
            skv.skv_attn_fwd_merged(plan, q, k, v, o, lse, ws, stream)
        else:
            skv.skv_attn_fwd(plan, q, k, v, ws, stream)
            skv.skv_lse_merge(plan, ws, o, lse, stream)
        status_log[2 * i:2 * i + 1].copy_(ws_status)
        if backward:
            skv.skv_attn_bwd(plan, q, k, v, o, lse, do, dq, dk, dv, ws, stream)
            status_log[2 * i + 1:2 * i + 2].copy_(ws_status)
        return plan

    def mk_event():
        e = torch.cuda.Event(enable_timing=True)
        e.record(stream)
        return e

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    planner_s.clear()

    K = steps
    ev = [(mk_event(), mk_event()) for _ in range(K)]
    kids = ((skv.SKV_KERNEL_FWD,) + (() if fused else (skv.SKV_KERNEL_MERGE,)) +
            ((skv.SKV_KERNEL_BWD,) if backward else ()))
    kev = {kid: [(mk_event(), mk_event()) for _ in range(K)] for kid in kids}
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # Inputs larger than L2 (K and V alone exceed it): the K steps run back to back
    # between one pair of events, the host planner of step i+1 overlapping step i on
    # the GPU as in a training loop. Smaller inputs: L2 flushed before every step,
    # outside that step's event window.
    kv_bytes = 2 * k.numel() * k.element_size()
    stream_mode = kv_bytes > L2_BYTES
    with ClockSampler(local_rank) as clocks:
        if stream_mode:
            ev[0][0].record(stream)
            for i in range(K):
                for kid, lst in kev.items():
                    skv.skv_set_timing_events(kid, lst[i][0], lst[i][1])
                step(warmup + i)
            ev[0][1].record(stream)
        else:
            for i in range(K):
                flush.zero_()
                for kid, lst in kev.items():
                    skv.skv_set_timing_events(kid, lst[i][0], lst[i][1])
                ev[i][0].record(stream)
                step(warmup + i)
                ev[i][1].record(stream)
        torch.cuda.synchronize()
    for kid in kev:
        skv.skv_set_timing_events(kid, None, None)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    bad = status_log.nonzero().flatten().tolist()
    if bad:
        codes = sorted(set(status_log.cpu().tolist()) - {0})
        raise RuntimeError(f"{name}: device status {codes} in step calls {bad} (warm-up and timed)")
    t_steps = [ev[0][0].elapsed_time(ev[0][1]) / 1e3] if stream_mode else [a.elapsed_time(b) / 1e3 for a, b in ev]
    t_kern = {kid: [a.elapsed_time(b) / 1e3 for a, b in lst] for kid, lst in kev.items()}
    total = max_over_ranks(sum(t_steps), world, dev)

    f_fwd_all, f_bwd_all, mbytes_all = 0.0, 0.0, 0.0
    for i in range(K):
        p = step_probs[warmup + i]
        a, b = flops_of(p, backward)
        f_fwd_all += a
        f_bwd_all += b
        if not fused:
            mbytes_all += merge_bytes(p, skv.skv_plan(p, policy, sizes=sizes[warmup + i]).stats()["n_fwd_units"])
    flops_rank = f_fwd_all + f_bwd_all
    value = job_value(sum_over_ranks(flops_rank, world, dev), total)
    ctx_tokens = sum_over_ranks(float(prob.num_tokens_kv) * K, world, dev)

    # plan quality (LPT vs static) on this step's problem
    p0 = step_probs[warmup]
    lpt = skv.skv_plan(p0, skv.SKV_PLAN_LPT).stats()["imbalance"]
    static = skv.skv_plan(p0, skv.SKV_PLAN_STATIC).stats()["imbalance"]

    realized = realized_busy_imbalance(skv, p0, policy, q, k, v, do, ws, o, lse, dq, dk, dv, stream, dev, fused)
    lpt_device = device_lpt_us(skv, p0, policy, dev, stream)

    peaks = load_peaks()
    kms = {kid: statistics.mean(t) for kid, t in t_kern.items()}

    def tensor_roof(kernel, flops_per_launch, t):
        a = flops_per_launch / t / 1e12
        return {"bound": "tensor", "kernel": kernel, "achieved": round(a, 2), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(a / peaks["bf16_tflops"], 4),
                "frac_of_sustained": (round(a / peaks["bf16_tflops_sustained"], 4)
                                      if peaks.get("bf16_tflops_sustained") else None),
                "traffic": profiled_traffic(kernel, name, setup),
                "peak_source": f"{peaks['source']} bf16 dense (burst)"}

    kernels = {"fwd": tensor_roof("fwd_kernel", f_fwd_all / K, kms[skv.SKV_KERNEL_FWD])}
    if fused:
        kernels["fwd"]["note"] = "forward with the LSE merge in its tail (one launch)"
    else:
        m_gbs = mbytes_all / K / kms[skv.SKV_KERNEL_MERGE] / 1e9
        kernels["merge"] = {"bound": "hbm", "kernel": "merge_kernel", "achieved": round(m_gbs, 1),
                            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(m_gbs / peaks["hbm_gbs"], 4),
                            "traffic": profiled_traffic("merge_kernel", name, setup),
                            "peak_source": f"{peaks['source']} HBM copy"}
    if backward:
        kernels["bwd"] = tensor_roof("bwd_kernel", f_bwd_all / K, kms[skv.SKV_KERNEL_BWD])
    roofline = dict(kernels["bwd" if backward else "fwd"])
    roofline["step_frac"] = round(flops_rank / K / (peaks["bf16_tflops"] * 1e12) / (total / K), 4)
    # forward: plan upload, forward (+ merge); backward: plan upload, prep, backward, dQ cast
    kernels_per_step = (2 if fused else 3) + (4 if backward else 0)

    rec = {
        "workload": f"{name}: {WORKLOAD_TEXT[name]}", "value": round(value, 3), "unit": "TFLOP/s", "steps": K,
        "warmup": warmup, "ms_per_step": round(total / K * 1e3, 4), "seed": args.seed, "policy": args.policy,
        "sub_chunks": prob.sub_chunks, "partials": args.partials, "queues": args.queues,
        "l2": (f"inputs larger than L2 (K+V {kv_bytes / 2**20:.0f} MiB > 126 MB): no flush, {K} steps back "
               "to back between two events, host planning of the next step overlapping the GPU")
              if stream_mode else "flushed before every step (256 MiB write outside the step's event window)",
        "roofline": roofline, "kernels": kernels,
        "kernel_ms": {"fwd": round(kms[skv.SKV_KERNEL_FWD] * 1e3, 4),
                      "merge": None if fused else round(kms[skv.SKV_KERNEL_MERGE] * 1e3, 4),
                      "bwd": round(kms[skv.SKV_KERNEL_BWD] * 1e3, 4) if backward else None},
        "merge": "in the forward kernel's tail" if fused else "separate launch",
        "context_tokens_per_s": round(ctx_tokens / total, 1),
        "imbalance": {"lpt": lpt, "static": static, "realized": realized},
        "planner_us": round(statistics.median(planner_s) * 1e6, 1),
        "lpt_device_us": lpt_device,
        "gpu_launches": kernels_per_step * K,
        "clocks": clocks.summary(),
    }
    if e2e:
        rec["e2e"] = run_e2e(args, prob, step_probs, sizes, policy, q, k, v, do, dev, world)
    del ws, flush, q, k, v, do, o, lse, dq, dk, dv
    torch.cuda.empty_cache()
    return rec, prob


def run_gpu(args, rank, world, local_rank):
    rec, prob = run_workload(args, args.workload, args.steps, args.warmup, rank, world, local_rank, not args.no_e2e)
    out = {
        "metric": METRIC, "value": rec["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": rec["steps"],
        "warmup": rec["warmup"], "ms_per_step": rec["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": rec["workload"], "seed": args.seed, "policy": args.policy,
                   "sub_chunks": rec["sub_chunks"], "partials": rec["partials"], "queues": rec["queues"],
                   "l2": rec["l2"],
                   "parallelism": f"replicas x{world}" if world > 1 else "1 GPU, P virtual partitions"},
    }
    for key in ("roofline", "kernels", "kernel_ms", "merge", "context_tokens_per_s", "imbalance", "planner_us",
                "lpt_device_us",
                "gpu_launches", "clocks", "e2e"):
        if key in rec:
            out[key] = rec[key]
    if world == 1 and not args.no_extra:
        # the other target workloads, each timed on its own (same contract: warm-up, then steps timed with
        # CUDA events, clocks sampled during its timed region)
        out["workloads"] = {}
        for name, sub in EXTRA_WORKLOADS:
            if name == args.workload and sub is None:
                continue
            r, _ = run_workload(args, name, min(args.steps, 20), args.warmup, rank, world, local_rank, False, sub)
            out["workloads"][name if sub is None else f"{name}_sub{sub}"] = r
    return out, prob


def device_lpt_us(skv, prob, policy, dev, stream):
    """The LPT placement of the step plan's items on the GPU (skv_lpt_place_device,
    one CTA): device time per launch, 20 launches back to back between two CUDA
    events on the launch stream, queued behind a 1 ms spin so that no host
    latency falls between them; median of 5 such runs. Checked against the
    host plan's partitions. None beyond its size limits."""
    plan = skv.skv_plan(prob, policy)
    it = plan.items()
    P = prob.num_partitions
    if len(it) > 16384 or P > 4096 or (policy & 0xff) == skv.SKV_PLAN_STATIC:
        return None
    costs = torch.from_numpy(it["cost"].astype(np.int64)).to(dev)
    part = torch.empty(len(it), dtype=torch.int32, device=dev)
    loads = torch.empty(P, dtype=torch.int64, device=dev)
    skv.skv_lpt_place_device(costs, P, part, loads, stream)  # warm-up
    times = []
    with torch.cuda.stream(stream):
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda._sleep(2_000_000)
            a.record(stream)
            for _ in range(20):
                skv.skv_lpt_place_device(costs, P, part, loads, stream)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b) * 1e3 / 20)
    if not np.array_equal(part.cpu().numpy(), it["partition"]):
        raise RuntimeError("device LPT placement differs from the host plan")
    return round(statistics.median(times), 1)


def realized_busy_imbalance(skv, prob, policy, q, k, v, do, ws, o, lse, dq, dk, dv, stream, dev, fused=True):
    """One more (untimed) step with the unit timer on: every work unit's
    %globaltimer start and end, summed per virtual partition, gives the realized
    busy time of each partition; its imbalance (max / mean - 1, mean over all P)
    is the measured counterpart of the plan's LPT imbalance."""
    backward = do is not None
    plan = skv.skv_plan(prob, policy)
    st = plan.stats()
    n_f, n_b = st["n_fwd_units"], st["n_bwd_units"]
    fst = torch.zeros(2 * max(n_f, 1), dtype=torch.int64, device=dev)
    bst = torch.zeros(2 * max(n_b, 1), dtype=torch.int64, device=dev)
    skv.skv_set_unit_timer(fst, bst if backward else None)
    try:
        if fused:
            skv.skv_attn_fwd_merged(plan, q, k, v, o, lse, ws, stream)
        else:
            skv.skv_attn_fwd(plan, q, k, v, ws, stream)
            skv.skv_lse_merge(plan, ws, o, lse, stream)
        if backward:
            skv.skv_attn_bwd(plan, q, k, v, o, lse, do, dq, dk, dv, ws, stream)
        torch.cuda.synchronize()
    finally:
        skv.skv_set_unit_timer(None, None)
    if skv.skv_status(ws) != 0:
        raise RuntimeError("device status error in the unit-timer step")
    fp, bp = plan.unit_partitions()
    P = prob.num_partitions

    def busy(stamps, parts, n):
        s = stamps.cpu().numpy()[:2 * n].reshape(n, 2).astype(np.float64)
        return np.bincount(parts, weights=s[:, 1] - s[:, 0], minlength=P)

    def imb(x):
        return round(float(x.max() / x.mean() - 1.0), 5) if x.mean() > 0 else None

    bf = busy(fst, fp, n_f)
    out = {"fwd": imb(bf)}
    if backward:
        bb = busy(bst, bp, n_b)
        out["bwd"] = imb(bb)
        out["fwd+bwd"] = imb(bf + bb)
    out["how"] = "sum of work-unit durations (%globaltimer) per virtual partition, one untimed step"
    return out


def run_e2e(args, prob, step_probs, sizes, policy, q, k, v, do, dev, world):
    """Same metric through the public API from pinned host buffers: every step
    copies its inputs host->device, runs the path and reads all its outputs
    back. Measured twice over the same steps:
      * pipelined (the reported value), as a training loop feeds data: inputs
        are copied in on one stream, outputs copied out on another, the path
        runs on a third, with two device buffer sets, so step i+1's inputs and
        step i-1's outputs move while step i computes;
      * serial: copy in, compute, copy out, one after the other."""
    from split_kv_block_b200 import skv
    backward = do is not None
    hin = {"q": q.cpu().pin_memory(), "k": k.cpu().pin_memory(), "v": v.cpu().pin_memory()}
    if backward:
        hin["do"] = do.cpu().pin_memory()
    Nq, Hq, d = prob.num_tokens_q, prob.num_q_heads, prob.head_dim
    NB = 2

    def out_set():
        o = {"o": torch.empty(Nq, Hq, d, dtype=torch.bfloat16, device=dev),
             "lse": torch.empty(Nq, Hq, dtype=torch.float32, device=dev)}
        if backward:
            o.update(dq=torch.empty_like(q), dk=torch.empty_like(k), dv=torch.empty_like(v))
        return o

    din = [{n: torch.empty_like(t, device=dev) for n, t in hin.items()} for _ in range(NB)]
    dout = [out_set() for _ in range(NB)]
    hout = {n: torch.empty(t.shape, dtype=t.dtype).pin_memory() for n, t in dout[0].items()}
    ws = torch.empty(max(s.ws_bytes for s in sizes), dtype=torch.uint8, device=dev)
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = sum(t.numel() * t.element_size() for t in hout.values())
    n = min(args.steps, args.e2e_steps)
    s_comp = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def compute(i, b, stream):
        p = step_probs[i % len(step_probs)]
        plan = skv.skv_plan(p, policy, sizes=sizes[i % len(sizes)])
        x, y = din[b], dout[b]
        if args.fused_merge:
            skv.skv_attn_fwd_merged(plan, x["q"], x["k"], x["v"], y["o"], y["lse"], ws, stream)
        else:
            skv.skv_attn_fwd(plan, x["q"], x["k"], x["v"], ws, stream)
            skv.skv_lse_merge(plan, ws, y["o"], y["lse"], stream)
        if backward:
            skv.skv_attn_bwd(plan, x["q"], x["k"], x["v"], y["o"], y["lse"], x["do"], y["dq"], y["dk"], y["dv"],
                             ws, stream)
        return p

    def run(first, count, pipelined):
        ev = lambda: torch.cuda.Event(enable_timing=True)
        in_done, comp_done, out_done = [ev() for _ in range(NB)], [ev() for _ in range(NB)], [ev() for _ in range(NB)]
        start, end = ev(), ev()
        torch.cuda.synchronize()
        start.record(s_comp)
        s_in.wait_stream(s_comp)
        s_out.wait_stream(s_comp)
        flops = 0.0
        for j in range(count):
            i, b = first + j, (j % NB) if pipelined else 0
            cin, cout = (s_in, s_out) if pipelined else (s_comp, s_comp)
            if pipelined and j >= NB:
                cin.wait_event(comp_done[b])       # step j-2 no longer reads din[b]
            with torch.cuda.stream(cin):
                for nme, t in hin.items():
                    din[b][nme].copy_(t, non_blocking=True)
            in_done[b].record(cin)
            if pipelined:
                s_comp.wait_event(in_done[b])
                if j >= NB:
                    s_comp.wait_event(out_done[b])  # step j-2's outputs have left dout[b]
            p = compute(i, b, s_comp)
            comp_done[b].record(s_comp)
            if pipelined:
                cout.wait_event(comp_done[b])
            with torch.cuda.stream(cout):
                for nme, t in hout.items():
                    t.copy_(dout[b][nme], non_blocking=True)
            out_done[b].record(cout)
            ff, fb = flops_of(p, backward)
            flops += ff + fb
        s_comp.wait_stream(s_in)
        s_comp.wait_stream(s_out)
        end.record(s_comp)
        end.synchronize()
        return start.elapsed_time(end) / 1e3, flops

    run(0, args.warmup, True)
    t_pipe, flops = run(args.warmup, n, True)
    t_ser, _ = run(args.warmup, n, False)
    t_pipe = max_over_ranks(t_pipe, world, dev)
    t_ser = max_over_ranks(t_ser, world, dev)
    flops_all = sum_over_ranks(flops, world, dev)
    return {"value": round(job_value(flops_all, t_pipe), 4), "unit": "TFLOP/s", "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h), "steps": n, "ms_per_step": round(t_pipe / n * 1e3, 3),
            "how": "pinned host buffers; copy-in, compute and copy-out on three streams, two device buffer sets",
            "serial": {"value": round(job_value(flops_all, t_ser), 4), "ms_per_step": round(t_ser / n * 1e3, 3)}}


# ------------------------------------------------------------- CPU oracle
def oracle_sample(prob, groups, anchor_stride):
    """Sub-problem: the kv-head groups `groups` and every `anchor_stride`-th
    anchor of each sample (exact for those rows and heads: rows and heads are
    independent)."""
    G = prob.num_q_heads // prob.num_kv_heads
    qh = [g * G + i for g in groups for i in range(G)]
    keep = []
    aoff = [0]
    for b in range(prob.num_samples):
        j = list(range(int(prob.anchor_offsets[b]), int(prob.anchor_offsets[b + 1])))[::anchor_stride]
        keep += j
        aoff.append(aoff[-1] + len(j))
    sub = prob.replace(num_q_heads=len(qh), num_kv_heads=len(groups), anchors=prob.anchors[keep],
                       anchor_offsets=np.array(aoff, dtype=np.int32))
    return sub, qh, keep


def time_oracle(prob, q, k, v, do, groups, anchor_stride):
    from oracle import attention as A
    sub, qh, keep = oracle_sample(prob, groups, anchor_stride)
    S = prob.block_q
    rows = np.concatenate([np.arange(j * S, (j + 1) * S) for j in keep]) if keep else np.zeros(0, dtype=np.int64)
    rows_t = torch.from_numpy(rows)
    qs = q[rows_t][:, qh].contiguous()
    ks, vs = k[:, list(groups)].contiguous(), v[:, list(groups)].contiguous()
    t0 = time.perf_counter()
    O, L = A.attention_forward(sub, qs, ks, vs)
    if do is not None:
        dos = do[rows_t][:, qh].contiguous()
        A.attention_backward(sub, qs, ks, vs, O, L, dos)
    dt = time.perf_counter() - t0
    ff, fb = flops_of(sub, do is not None)
    return (ff + fb), dt, sub


def cpu_baseline(prob, backward, seed):
    q, k, v, do = synth.make_tensors(prob, seed=seed, backward=backward)
    threads = os.cpu_count() or 1
    torch.set_num_threads(threads)
    # calibrate on one kv-head group and every 8th anchor, then take as many
    # groups / anchors as make ~15 s of CPU work (heads and rows are independent)
    f, dt, sub = time_oracle(prob, q, k, v, do if backward else None, (0,), 8)
    per_group_all = dt * 8
    n_groups = max(1, min(prob.num_kv_heads, int(15.0 / max(per_group_all, 1e-3))))
    stride = 1 if per_group_all <= 15.0 else int(math.ceil(per_group_all / 15.0))
    groups = tuple(range(n_groups))
    f, dt, sub = time_oracle(prob, q, k, v, do if backward else None, groups, stride)
    # a sample shorter than ~10 s (the whole workload fits) is run again until it is not
    reps = 1
    while dt < 10.0:
        f1, dt1, _ = time_oracle(prob, q, k, v, do if backward else None, groups, stride)
        f, dt, reps = f + f1, dt + dt1, reps + 1
    from oracle import planner as PL
    t0 = time.perf_counter()
    PL.lpt_plan(prob)
    lpt_s = time.perf_counter() - t0
    return {"value": round(f / dt / 1e12, 6), "unit": "TFLOP/s", "cores": torch.get_num_threads(), "kind": "oracle",
            "sample": f"fp64 oracle fwd{'+bwd' if backward else ''} on {n_groups} of {prob.num_kv_heads} kv-head "
                      f"groups, every {stride}th anchor ({int(sub.anchor_offsets[-1])} anchors), run {reps}x, "
                      f"{dt:.1f} s",
            "lpt_planner_us": round(lpt_s * 1e6, 1),
            "cpu": _cpu_name()}


def _cpu_name():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args):
    """The oracle as the reference arm: every step a bounded sample of the workload."""
    w = synth.WORKLOADS[args.workload]
    prob = synth.make_problem(w, seed=args.seed, sub_chunks=args.sub_chunks)
    backward = w.backward
    q, k, v, do = synth.make_tensors(prob, seed=args.seed, backward=backward)
    torch.set_num_threads(os.cpu_count() or 1)
    n_anchor = int(prob.anchor_offsets[-1])
    # calibrate: one group, a thin anchor sample
    f, dt, _ = time_oracle(prob, q, k, v, do if backward else None, (0,), max(1, n_anchor // 2))
    budget = min(5.0, 150.0 / max(1, args.steps + args.warmup))
    per_anchor = dt / max(1, len(range(0, n_anchor, max(1, n_anchor // 2))))
    n_take = max(1, min(n_anchor, int(budget / max(per_anchor, 1e-6))))
    stride = max(1, n_anchor // n_take)
    times, flops = [], 0.0
    for i in range(args.warmup + args.steps):
        g = i % prob.num_kv_heads
        f, dt, sub = time_oracle(prob, q, k, v, do if backward else None, (g,), stride)
        if i >= args.warmup:
            times.append(dt)
            flops += f
    total = sum(times)
    value = flops / total / 1e12
    sample = (f"fp64 oracle fwd{'+bwd' if backward else ''} per step on one kv-head group (rotating) and every "
              f"{stride}th anchor of the workload")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(total / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{args.workload}: {WORKLOAD_TEXT[args.workload]}", "seed": args.seed,
                   "policy": args.policy, "sub_chunks": prob.sub_chunks, "parallelism": "CPU host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": torch.get_num_threads(),
                         "kind": "oracle", "sample": sample, "cpu": _cpu_name()},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="skv", choices=["skv", "reference"])
    ap.add_argument("--workload", default="ctx32k", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--policy", default="lpt", choices=["lpt", "static", "lpt_tiles"])
    ap.add_argument("--sub-chunks", type=int, default=None)
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="time the headline workload only")
    ap.add_argument("--queues", default="one", choices=["one", "partition"],
                    help="work queues of the kernels: one for all items (default), or one per partition "
                         "(SKV_PLAN_PARTITION_QUEUES)")
    ap.add_argument("--partials", default="fp32", choices=["fp32", "bf16"],
                    help="storage of the per-chunk partial outputs between the forward and the merge")
    ap.add_argument("--fused-merge", action="store_true",
                    help="run the LSE merge in the forward kernel's tail (skv_attn_fwd_merged) instead of as its own "
                         "launch")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    check_world(args.gpus, world)

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        out, prob = run_gpu(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not args.no_cpu_baseline:
                out["cpu_baseline"] = cpu_baseline(prob, synth.WORKLOADS[args.workload].backward, args.seed)
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
