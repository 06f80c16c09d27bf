"""split_kv_block_b200 — split-KV block-sparse cross-attention for B200 (sm_100a).

    from split_kv_block_b200 import skv      # C-ABI binding (needs libskv.so)
    from split_kv_block_b200 import synth    # seeded synthetic workloads

Build the CUDA library with `python -m split_kv_block_b200.build`.
"""
__all__ = ["skv", "synth", "build"]
