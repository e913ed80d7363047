"""B200-native NVFP4 MoE train/rollout alignment hot path.

The compute lives in ``libquads.so`` (hand-written sm_100a CUDA behind a C
ABI declared in ``include/quads.h``); ``binding`` marshals torch tensors to
it.  Importing this package does not load the library; the first call does,
and raises if it is missing.
"""
__all__ = ["binding", "workloads"]
