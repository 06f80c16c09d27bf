"""CPU oracle for split-KV attention — test infrastructure, not product code.

A plain, slow, fp64 restatement of what the split-KV hot path computes, used
only to check the CUDA path: the tests under tests/, the package smoke check
(__graft_entry__.smoke) and the CPU baseline leg of bench.py may import it;
nothing in the product path does, and the product fails loudly rather than
fall back to it. It shares no code with the CUDA path; both take their inputs
from split_kv_block_b200.synth, which holds no arithmetic of the method.

Sources (web pages on the method):
  [Abstract]  "Split-KV: Efficient Context Parallelism for Training Diffusion
              Drafters" (arXiv 2611.05926), Abstract.
  [Article]   "Split-KV: Breaking the Context Parallelism Bottleneck in
              Diffusion Drafter Training", sections "The Query-Context
              Asymmetry", "Split-KV's Core Mechanism: Decoupling Communication
              from Context Length", "LPT Scheduling: Load Balancing with Real
              Attention Costs".

Modules:
  attention  masked cross-attention forward/backward (the unsplit definition),
             per-chunk partials and the exact log-sum-exp merge, the chunked
             backward.
  planner    work items, realized cost, LPT, the static token split,
             imbalance.

Every function is pinned by tests/test_oracle_*.py against closed forms,
library routines, brute force or textbook instances; none is "parity
unpinned".
"""
from . import attention, planner  # noqa: F401
