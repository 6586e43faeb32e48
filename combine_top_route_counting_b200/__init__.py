"""Deterministic MoE layer forward on B200 (sm_100a): top-k routing, the
counting-sort pull-dispatch schedule Phi, gather into per-expert buffers, a
grouped SwiGLU expert FFN on tcgen05 tensor cores, and a fixed-order combine.

The compute lives in a C-ABI shared library (libmoe_b200.so, built from
csrc/); `moe` is its thin Python binding and `inputs` the seeded workload
generators.
"""
__all__ = ["moe", "inputs"]
