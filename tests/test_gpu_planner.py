"""The LPT placement on the device (skv_lpt_place_device) against the host
planner's, through the C ABI: for the items of every benchmark workload
(their realized costs, and the executed-tile costs), the device kernel's
partition of every item and the partition loads equal skv_plan's bit for bit
("Split-KV: Breaking the Context Parallelism Bottleneck in Diffusion Drafter
Training", section "LPT Scheduling")."""
import numpy as np
import pytest
import torch

from split_kv_block_b200 import skv, synth

pytestmark = pytest.mark.gpu


def _device_place(plan):
    it = plan.items()
    costs = torch.from_numpy(it["cost"].astype(np.int64)).cuda()
    P = plan.problem.num_partitions
    part = torch.full((len(it),), -1, dtype=torch.int32, device="cuda")
    loads = torch.empty(P, dtype=torch.int64, device="cuda")
    skv.skv_lpt_place_device(costs, P, part, loads)
    torch.cuda.synchronize()
    return it, part.cpu().numpy(), loads.cpu().numpy()


@pytest.mark.parametrize("name,sub", [("tiny_4k", None), ("ctx32k", None), ("ctx128k", 1), ("ctx128k", 4),
                                      ("batch8_logu", None), ("ctx32k_sparse", None)])
def test_device_lpt_equals_host_lpt(name, sub):
    prob = synth.make_problem(synth.WORKLOADS[name], seed=0, sub_chunks=sub)
    for policy in (skv.SKV_PLAN_LPT, skv.SKV_PLAN_LPT_TILES):
        if policy == skv.SKV_PLAN_LPT_TILES and name == "batch8_logu":
            continue  # same placement code; the tile costs of 8 samples take long on the host only
        plan = skv.skv_plan(prob, policy)
        it, part, loads = _device_place(plan)
        assert np.array_equal(part, it["partition"])
        assert np.array_equal(loads, plan.partition_load)


def test_device_lpt_edge_cases():
    """Ties everywhere (equal costs: the lower index first, the lower
    partition first), zero costs, one item, more partitions than items."""
    for costs, P in (([5] * 37, 4), ([0] * 10, 3), ([7], 5), ([3, 3, 2, 2, 2], 2), ([9, 1, 9, 1, 0, 4], 8)):
        c = torch.tensor(costs, dtype=torch.int64, device="cuda")
        part = torch.empty(len(costs), dtype=torch.int32, device="cuda")
        loads = torch.empty(P, dtype=torch.int64, device="cuda")
        skv.skv_lpt_place_device(c, P, part, loads)
        torch.cuda.synchronize()
        # the host reference: sorted by (cost desc, index), smallest (load, partition)
        order = sorted(range(len(costs)), key=lambda i: (-costs[i], i))
        ld = [0] * P
        ref = [0] * len(costs)
        for i in order:
            p = min(range(P), key=lambda x: (ld[x], x))
            ref[i] = p
            ld[p] += costs[i]
        assert part.cpu().tolist() == ref and loads.cpu().tolist() == ld


def _host_lpt(costs, P):
    """Sorted by (cost desc, index); each item to the smallest (load, partition)."""
    import heapq
    heap = [(0, p) for p in range(P)]
    part = [0] * len(costs)
    for i in sorted(range(len(costs)), key=lambda i: (-costs[i], i)):
        ld, p = heapq.heappop(heap)
        part[i] = p
        heapq.heappush(heap, (ld + costs[i], p))
    loads = [0] * P
    for ld, p in heap:
        loads[p] = ld
    return part, loads


@pytest.mark.parametrize("n,P,scale", [(0, 3, 10), (1000, 1, 10), (1000, 17, 10), (777, 33, 10**6), (2000, 64, 3),
                                       (1248, 128, 10**9), (3000, 129, 10**9), (16384, 1000, 10**4),
                                       (5000, 4096, 10**7), (300, 40, 2**50), (300, 200, 2**60)])
def test_device_lpt_every_path(n, P, scale):
    """Every placement path of the kernel: keys packed with the loads in
    registers (up to 32, 64 and 128 partitions) or in shared memory (more
    partitions), and unpacked when a cost or the costs' sum reaches 2^51;
    the item and partition limits; random costs with many ties."""
    rng = np.random.default_rng(n * 7 + P)
    costs = rng.integers(0, scale, size=n, dtype=np.int64) if n else np.zeros(0, dtype=np.int64)
    c = torch.from_numpy(costs).cuda() if n else torch.zeros(1, dtype=torch.int64, device="cuda")
    part = torch.full((max(n, 1),), -1, dtype=torch.int32, device="cuda")
    loads = torch.empty(P, dtype=torch.int64, device="cuda")
    L = skv.lib()
    import ctypes
    assert L.skv_lpt_place_device(ctypes.c_void_p(c.data_ptr()), n, P, ctypes.c_void_p(part.data_ptr()),
                                  ctypes.c_void_p(loads.data_ptr()), None) == 0
    torch.cuda.synchronize()
    ref_part, ref_loads = _host_lpt(costs.tolist(), P)
    assert part.cpu().tolist()[:n] == ref_part
    assert loads.cpu().tolist() == ref_loads
