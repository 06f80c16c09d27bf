"""Writes the stored expected values under tests/golden/ from the CPU oracle
only (no CUDA path involved). Run from the repository root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import planner as PL  # noqa: E402
from split_kv_block_b200 import synth  # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def tiny_plan():
    prob = synth.make_problem(synth.WORKLOADS["tiny_4k"], seed=0)
    items, loads = PL.lpt_plan(prob)
    s_items, s_loads = PL.static_plan(prob)
    return {
        "workload": "tiny_4k (1 sample, 4096-token context, 4 anchors x 16 tokens, 8/2 heads, d=64, "
                    "chunk 512, 4 partitions), seed 0",
        "anchors": prob.anchors.tolist(),
        "lpt_items": [[it.b, it.c, it.g, it.sub, it.key_begin, it.key_end, it.cost, it.partition] for it in items],
        "lpt_loads": loads,
        "lpt_imbalance": PL.imbalance(loads),
        "static_loads": s_loads,
        "static_imbalance": PL.imbalance(s_loads),
    }


if __name__ == "__main__":
    g = tiny_plan()
    lines = ["{"]
    keys = list(g)
    for i, k in enumerate(keys):
        end = "," if i + 1 < len(keys) else ""
        if k == "lpt_items":
            rows = ",\n  ".join(json.dumps(r) for r in g[k])
            lines.append(f' "{k}": [\n  {rows}\n ]{end}')
        else:
            lines.append(f" {json.dumps(k)}: {json.dumps(g[k])}{end}")
    lines.append("}")
    with open(os.path.join(HERE, "tiny_4k_plan.json"), "w") as f:
        f.write("\n".join(lines) + "\n")
    print("wrote tiny_4k_plan.json")
