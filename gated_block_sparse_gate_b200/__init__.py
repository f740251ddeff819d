"""gated_block_sparse_gate_b200: gated block-sparse causal attention on B200.

The compute lives in ``libgbs.so`` (hand-written sm_100a CUDA behind a C ABI,
declared in ``include/gbs.h``). ``binding`` marshals torch tensors into that
ABI; ``inputs`` draws the seeded synthetic workloads.
"""
