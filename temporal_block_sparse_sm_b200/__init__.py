"""B200-native LiteAttention: temporally sparse attention with a persistent skip mask.

The compute path is the CUDA library ``libliteattn.so`` (sm_100a), reached
through the ctypes binding in :mod:`temporal_block_sparse_sm_b200.liteattn`.
Importing this package does not load the library; the first call that needs
it does, and raises if it is missing.

Modules: ``liteattn`` (the C ABI and the Plan / Mask objects), ``propagation``
(mask propagation policies), ``calibration`` (per-step thresholds from error
budgets), ``host_pipeline`` (steps on host-resident tensors with overlapped
copies), ``synthetic`` (seeded video-token workloads).
"""
__all__ = ["liteattn", "synthetic", "propagation", "calibration", "host_pipeline"]
