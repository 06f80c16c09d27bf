"""Host-side arithmetic of bench.py, on CPU: the FLOP count that every
throughput figure divides by, the algorithmic bytes of the backward roofline,
the lookup of ncu traffic by source digest, and the summary of the clock
samples that decides whether a run is kept."""
import json
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from split_kv_block_b200 import skv, synth  # noqa: E402


@pytest.mark.parametrize("name", ["tiny_4k", "ctx32k", "ctx32k_sparse"])
def test_flops_match_the_planners_unmasked_count(name):
    """4 d per unmasked (token, key, q-head) triple forward, 2.5x that backward; the
    planner counts the triples independently (its realized item costs)."""
    prob = synth.make_problem(synth.WORKLOADS[name], seed=0)
    f_fwd, f_bwd = bench.flops_of(prob, True)
    triples = skv.skv_plan(prob).stats()["total_cost"]
    assert f_fwd == 4.0 * prob.head_dim * triples
    assert f_bwd == 2.5 * f_fwd
    assert bench.flops_of(prob, False)[1] == 0.0


def test_flops_of_a_hand_problem():
    # two samples, anchors 5, 9 and 3; block_q 2, 4 q-heads, d 8: 4*8*2*4*(5+9+3)
    prob = synth.small_problem([10, 4], [[5, 9], [3]], block_q=2, hq=4, hkv=2, d=8)
    assert bench.flops_of(prob)[0] == 4 * 8 * 2 * 4 * 17


def test_backward_bytes_by_hand():
    """Q, dO bf16 read; LSE, D fp32 read; K/V of each sample's attended prefix
    read and dK/dV of it written (bf16); dQ fp32 read and written."""
    prob = synth.small_problem([10, 4], [[5, 9], [3]], block_q=2, hq=4, hkv=2, d=8)
    nq = 3 * 2  # three anchors of two tokens
    rows = nq * 4
    keys = 9 + 3  # largest anchor per sample
    expect = 2 * rows * 8 * 2 + 2 * rows * 4 + 4 * keys * 2 * 8 * 2 + 2 * rows * 8 * 4
    assert bench.bwd_bytes(prob) == expect


def test_job_value_is_total_work_over_the_slowest_rank():
    assert bench.job_value(6e12, 2.0) == pytest.approx(3.0)


def _fake_root(tmp_path, records):
    """A repository root whose sources are the real kernel sources and whose
    traffic record is the one given."""
    os.makedirs(tmp_path / "split_kv_block_b200")
    os.symlink(os.path.join(ROOT, "split_kv_block_b200", "csrc"), tmp_path / "split_kv_block_b200" / "csrc")
    os.makedirs(tmp_path / "profiles")
    with open(tmp_path / "profiles" / "dram_traffic.json", "w") as f:
        json.dump(records, f)
    return str(tmp_path)


def test_traffic_is_reported_only_for_the_captured_sources(tmp_path, monkeypatch):
    digest = bench.kernel_digest("bwd_kernel")
    root = _fake_root(tmp_path, {"bwd_kernel": {"ctx32k": {"source_digest": digest, "dram_bytes_per_launch": 123},
                                                "ctx128k": {"source_digest": "0" * 16, "dram_bytes_per_launch": 7}}})
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.kernel_digest("bwd_kernel") == digest
    assert bench.profiled_traffic("bwd_kernel", "ctx32k") == 123
    assert bench.profiled_traffic("bwd_kernel", "ctx128k") is None  # kernel changed since that capture
    assert bench.profiled_traffic("bwd_kernel", "batch8_logu") is None  # never captured
    assert bench.profiled_traffic("fwd_kernel", "ctx32k") is None


def test_traffic_is_reported_only_for_the_captured_setup(tmp_path, monkeypatch):
    digest = bench.kernel_digest("fwd_kernel")
    setup = {"policy": "lpt", "partials": "fp32", "queues": "partition", "merge": "separate", "sub_chunks": 1}
    root = _fake_root(tmp_path, {"fwd_kernel": {"ctx32k": {"source_digest": digest, "dram_bytes_per_launch": 5,
                                                           "setup": setup}}})
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.profiled_traffic("fwd_kernel", "ctx32k", dict(setup)) == 5
    for key, other in (("partials", "bf16"), ("queues", "one"), ("merge", "fused"), ("sub_chunks", 4)):
        assert bench.profiled_traffic("fwd_kernel", "ctx32k", {**setup, key: other}) is None


def test_digest_follows_every_listed_source(tmp_path, monkeypatch):
    """Editing any file of a kernel's source list changes its digest."""
    src = tmp_path / "split_kv_block_b200" / "csrc"
    os.makedirs(src)
    for name in bench.KERNEL_SOURCES["merge_kernel"]:
        (src / name).write_text(name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    before = bench.kernel_digest("merge_kernel")
    for name in bench.KERNEL_SOURCES["merge_kernel"]:
        (src / name).write_text(name + " edited")
        after = bench.kernel_digest("merge_kernel")
        assert after != before
        before = after


def _sampler(rows):
    s = bench.ClockSampler(0)
    s.rows = [[str(x) for x in r] for r in rows]
    return s


def test_clock_summary_median_under_load_and_reasons():
    na, act = "Not Active", "Active"
    rows = [[1965, 1965, 950, na, na, na, act],
            [1950, 1965, 990, na, na, na, act],
            [1965, 1965, 970, na, na, na, na],
            [345, 1965, 120, na, na, na, na]]  # idle sample before the load: not in the median
    out = _sampler(rows).summary()
    assert out["sm_mhz"] == 1965.0
    assert out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 4


def test_clock_summary_names_every_throttle_reason_seen():
    na, act = "Not Active", "Active"
    out = _sampler([[1500, 1965, 1000, act, na, act, na], [1400, 1965, 1000, na, act, na, na]]).summary()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
    assert out["sm_mhz"] == pytest.approx(1450.0)


def test_clock_summary_without_samples():
    out = bench.ClockSampler(0).summary()
    assert out["sm_mhz"] is None and out["reasons"] == ["unsampled"]


def test_merge_bytes_by_hand():
    """Partials read (fp32 row of d plus its LSE, 128 rows per forward unit),
    merged O (bf16) and LSE (fp32) written once."""
    prob = synth.small_problem([10, 4], [[5, 9], [3]], block_q=2, hq=4, hkv=2, d=8)
    rows = 3 * 2 * 4
    assert bench.merge_bytes(prob, 5) == 5 * 128 * 9 * 4 + rows * 8 * 2 + rows * 4


def test_gpus_flag_must_match_the_ranks():
    bench.check_world(1, 1)
    bench.check_world(4, 4)
    for gpus, world in ((2, 1), (1, 2), (0, 1)):
        with pytest.raises(SystemExit):
            bench.check_world(gpus, world)
