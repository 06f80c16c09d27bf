"""The N>1 host path of bench.py on CPU: two gloo ranks started the way
torchrun starts them (RANK / WORLD_SIZE / MASTER_ADDR=127.0.0.1). Multi-GPU runs
are replicas: every rank plans and runs its own problem (seed + rank), with no
data-path collective; the job time is the maximum of the ranks' device times and
the value is the work of all ranks over that time."""
import argparse
import datetime
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


def _worker(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        from split_kv_block_b200 import skv
        args = argparse.Namespace(seed=3, workload="ctx32k", sub_chunks=None)
        seed, prob = bench.rank_problem(args, rank)
        plan = skv.skv_plan(prob)  # each rank plans its own problem (host planner)
        flops = sum(bench.flops_of(prob, True))
        t_rank = 0.5 + 0.25 * rank  # this rank's device time
        cpu = torch.device("cpu")
        t_job = bench.max_over_ranks(t_rank, world, cpu)
        f_job = bench.sum_over_ranks(flops, world, cpu)
        np.save(os.path.join(out_dir, f"rank{rank}.npy"),
                np.array([seed, float(np.sum(prob.anchors)), plan.stats()["total_cost"], flops, t_job, f_job,
                          bench.job_value(f_job, t_job)], dtype=np.float64))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_max_time_and_summed_work(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True, start_method="spawn")
    r = [np.load(tmp_path / f"rank{i}.npy") for i in range(world)]
    seeds = [int(x[0]) for x in r]
    assert seeds == [3, 4]
    # independent problems: different anchors, so different work per rank
    assert r[0][1] != r[1][1]
    for i in range(world):
        # planned cost = unmasked pairs x q-heads per group; FLOPs = 4 d S Hq sum(a) (+2.5x backward)
        assert r[i][2] > 0
    for i in range(world):
        assert r[i][4] == pytest.approx(0.75)           # job time: the slowest rank
        assert r[i][5] == pytest.approx(r[0][3] + r[1][3])  # job work: every rank's own
        assert r[i][6] == pytest.approx((r[0][3] + r[1][3]) / 0.75 / 1e12)
